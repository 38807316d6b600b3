// decode.cu -- one decoding step of the DAM sparse attention.
//
// The extended mask is the same as for prefill (DAM review page, "What carries the
// argument": the kept patterns are pasted over the whole S x S square; Referee Report
// summary: the mask is applied to the scaled logits before the softmax).  At a
// decoding step the only new query of a sequence sits at position pos, so it attends
// to row pos of that mask: keys pos - r for every extended diagonal r <= pos and every
// extended column c <= pos, read from the sequence's key/value cache.  A key that is
// both (pos - r == c) counts once; as in the prefill plan, columns own such keys.
//
// With one query row per (sequence, head) the work is a sequence of dot products over
// gathered cache rows: bound by the HBM traffic of the key and value rows, not by the
// tensor cores (an M = 1 product), so it runs on the FMA pipe.
//
// Kernels
//   decode_partial_kernel  one CTA (4 warps) per (sequence, head, split): the split's
//                          slice of the head's key list (band keys, then columns); each
//                          warp resolves 32 keys at once (one lane each) and streams them
//                          in groups of 8; a lane holds d/32 dimensions, so every key and
//                          value row is read as one coalesced warp access;
//                          fp32 online softmax in the log2 domain; the 4 warps' partial
//                          (max, sum, O) are merged in shared memory and written out
//   decode_combine_kernel  one warp per (sequence, head): merges the splits' partials
//                          into O (bf16) and LSE (natural log)
#include <cuda_bf16.h>

#include "common.cuh"
#include "trace.h"

namespace ssa {
namespace {

constexpr int kMaxSplits = 16;
constexpr int kDecThreads = 128;
constexpr int kKeysPerIter = 8;

// Splits of each (sequence, head) key list: the smallest power of two (<= 16) that gives
// at least 1024 CTAs, enough to keep HBM busy (on the 16-sequence x 32-head step, 2
// splits measured fastest; 1 leaves too few CTAs, 4..16 give each warp too few keys).
int dec_splits(int B, int H) {
    const long long bh = static_cast<long long>(B) * H;
    int s = 1;
    while (s < kMaxSplits && bh * s < 1024) s <<= 1;
    return s;
}

struct DecParams {
    int B, H, Hkv, S, d, splits;
    const uint16_t *Q, *K, *V;
    const int32_t *pos;
    const int32_t *dptr, *doff, *vptr, *vcol;
    const int32_t *kv_map;
    float scale_log2;
    float *part;  // [B][H][splits][2 + d]: max (log2 domain), sum, O
    uint16_t *O;
    float *LSE;
    int32_t *status;
};

__device__ __forceinline__ int dec_kv_head(const DecParams &p, int h) {
    return p.kv_map ? __ldg(p.kv_map + h) : h / (p.H / p.Hkv);
}

// True iff x is in the ascending array a[0..n).
__device__ __forceinline__ bool contains(const int32_t *a, int n, int32_t x) {
    const int k = lower_bound_i32(a, n, x);
    return k < n && __ldg(a + k) == x;
}

// Loads DPL consecutive bf16 of a row at lane offset as floats.
template <int DPL>
__device__ __forceinline__ void load_row(const uint16_t *row, int lane, float (&x)[DPL]) {
    if constexpr (DPL == 4) {
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(row) + lane);
        x[0] = __uint_as_float(w.x << 16);
        x[1] = __uint_as_float(w.x & 0xffff0000u);
        x[2] = __uint_as_float(w.y << 16);
        x[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(row) + lane);
        x[0] = __uint_as_float(w << 16);
        x[1] = __uint_as_float(w & 0xffff0000u);
    }
}

template <int D, int SPLITS>
__global__ void __launch_bounds__(kDecThreads) decode_partial_kernel(DecParams p) {
    constexpr int DPL = D / 32;  // dimensions per lane
    __shared__ float s_part[kDecThreads / 32][2 + D];
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = dec_kv_head(p, h);
    const int pos = __ldg(p.pos + b);
    const bool bad = g < 0 || g >= p.Hkv || pos < 0 || pos >= p.S;
    if (bad && threadIdx.x == 0 && split == 0) report(p.status, SSA_ERR_INVALID);
    const int32_t *Dh = p.doff + __ldg(p.dptr + h);
    const int32_t *Ch = p.vcol + __ldg(p.vptr + h);
    const int nd = bad ? 0 : __ldg(p.dptr + h + 1) - __ldg(p.dptr + h);
    const int nc = bad ? 0 : __ldg(p.vptr + h + 1) - __ldg(p.vptr + h);
    // the head's key list: band entries 0..nd-1, then column entries nd..nd+nc-1
    const int total = nd + nc;
    const int lo = static_cast<int>(static_cast<long long>(total) * split / SPLITS);
    const int hi = static_cast<int>(static_cast<long long>(total) * (split + 1) / SPLITS);

    float q[DPL];
    load_row<DPL>(p.Q + (static_cast<size_t>(b) * p.H + h) * D, lane, q);
#pragma unroll
    for (int k = 0; k < DPL; ++k) q[k] *= p.scale_log2;
    const size_t cache = (static_cast<size_t>(b) * p.Hkv + (bad ? 0 : g)) * p.S;
    const uint16_t *Kc = p.K + cache * D, *Vc = p.V + cache * D;

    float m = -INFINITY, l = 0.0f, o[DPL];
#pragma unroll
    for (int k = 0; k < DPL; ++k) o[k] = 0.0f;
    // Each warp takes 32 entries of the key list at a time: lane t resolves entry e0 + t
    // (band: pos - r unless that key is a column; column: c if c <= pos; -1: none), so the
    // lookups run in parallel; the warp then streams the 32 keys in groups of 8.
    for (int e0 = lo + 32 * warp; e0 < hi; e0 += 32 * (kDecThreads / 32)) {
        int mine = -1;
        {
            const int e = e0 + lane;
            if (e < hi) {
                if (e < nd) {
                    const int r = __ldg(Dh + e);
                    if (r <= pos && (nc == 0 || !contains(Ch, nc, pos - r))) mine = pos - r;
                } else {
                    const int c = __ldg(Ch + e - nd);
                    if (c <= pos) mine = c;
                }
            }
        }
        if (!__any_sync(0xffffffffu, mine >= 0)) continue;
#pragma unroll 2
        for (int g0 = 0; g0 < 32; g0 += kKeysPerIter) {
            int key[kKeysPerIter];
#pragma unroll
            for (int t = 0; t < kKeysPerIter; ++t) key[t] = __shfl_sync(0xffffffffu, mine, g0 + t);
            float kx[kKeysPerIter][DPL], vx[kKeysPerIter][DPL];
#pragma unroll
            for (int t = 0; t < kKeysPerIter; ++t) {
                const int j = key[t] < 0 ? 0 : key[t];
                load_row<DPL>(Kc + static_cast<size_t>(j) * D, lane, kx[t]);
                load_row<DPL>(Vc + static_cast<size_t>(j) * D, lane, vx[t]);
            }
            float sc[kKeysPerIter];
#pragma unroll
            for (int t = 0; t < kKeysPerIter; ++t) {
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < DPL; ++k) acc = fmaf(q[k], kx[t][k], acc);
                sc[t] = acc;
            }
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) {
#pragma unroll
                for (int t = 0; t < kKeysPerIter; ++t) sc[t] += __shfl_xor_sync(0xffffffffu, sc[t], o2);
            }
            float gmax = -INFINITY;
#pragma unroll
            for (int t = 0; t < kKeysPerIter; ++t) {
                if (key[t] < 0) sc[t] = -INFINITY;
                gmax = fmaxf(gmax, sc[t]);
            }
            if (gmax == -INFINITY) continue;  // no key in this group
            const float m_new = fmaxf(m, gmax);
            const float corr = ex2_approx(m - m_new);  // m = -inf at first: 0
            l *= corr;
#pragma unroll
            for (int k = 0; k < DPL; ++k) o[k] *= corr;
            m = m_new;
#pragma unroll
            for (int t = 0; t < kKeysPerIter; ++t) {
                const float pr = ex2_approx(sc[t] - m);  // -inf -> 0
                l += pr;
#pragma unroll
                for (int k = 0; k < DPL; ++k) o[k] = fmaf(pr, vx[t][k], o[k]);
            }
        }
    }
    // merge the warps of the CTA
    float *wpart = s_part[warp];
    if (lane == 0) {
        wpart[0] = m;
        wpart[1] = l;
    }
#pragma unroll
    for (int k = 0; k < DPL; ++k) wpart[2 + DPL * lane + k] = o[k];
    __syncthreads();
    if (warp == 0) {
        float M = -INFINITY;
        for (int w = 0; w < kDecThreads / 32; ++w) M = fmaxf(M, s_part[w][0]);
        float L = 0.0f, acc[DPL];
#pragma unroll
        for (int k = 0; k < DPL; ++k) acc[k] = 0.0f;
        if (M != -INFINITY) {
            for (int w = 0; w < kDecThreads / 32; ++w) {
                const float f = ex2_approx(s_part[w][0] - M);
                L += s_part[w][1] * f;
#pragma unroll
                for (int k = 0; k < DPL; ++k) acc[k] = fmaf(s_part[w][2 + DPL * lane + k], f, acc[k]);
            }
        }
        float *out = p.part + ((static_cast<size_t>(b) * p.H + h) * SPLITS + split) * (2 + D);
        if (lane == 0) {
            out[0] = M;
            out[1] = L;
        }
#pragma unroll
        for (int k = 0; k < DPL; ++k) out[2 + DPL * lane + k] = acc[k];
    }
}

template <int D, int SPLITS>
__global__ void __launch_bounds__(128) decode_combine_kernel(DecParams p) {
    constexpr int DPL = D / 32;
    const int item = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (item >= p.B * p.H) return;
    const float *part = p.part + static_cast<size_t>(item) * SPLITS * (2 + D);
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < SPLITS; ++k) M = fmaxf(M, part[k * (2 + D)]);
    float L = 0.0f, acc[DPL];
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[k] = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
        for (int k = 0; k < SPLITS; ++k) {
            const float *pk = part + k * (2 + D);
            const float f = ex2_approx(pk[0] - M);
            L += pk[1] * f;
#pragma unroll
            for (int t = 0; t < DPL; ++t) acc[t] = fmaf(pk[2 + DPL * lane + t], f, acc[t]);
        }
    }
    // no retained key: O = 0, LSE = -inf
    const bool empty = !(M > -INFINITY) || !(L > 0.0f);
    const float inv = empty ? 0.0f : 1.0f / L;
    uint16_t *orow = p.O + static_cast<size_t>(item) * D + DPL * lane;
#pragma unroll
    for (int t = 0; t < DPL; t += 2) {
        const __nv_bfloat162 v2 = __floats2bfloat162_rn(acc[t] * inv, acc[t + 1] * inv);
        *reinterpret_cast<__nv_bfloat162 *>(orow + t) = v2;
    }
    if (lane == 0) p.LSE[item] = empty ? -INFINITY : (M + log2f(L)) * 0.69314718055994531f;
}

template <int D, int SPLITS>
int launch_decode_s(DecParams &p, cudaStream_t s) {
    dim3 grid(SPLITS, p.H, p.B);
    decode_partial_kernel<D, SPLITS><<<grid, kDecThreads, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    decode_combine_kernel<D, SPLITS><<<(p.B * p.H + 3) / 4, 128, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    return SSA_OK;
}

template <int D>
int launch_decode(DecParams &p, cudaStream_t s) {
    switch (p.splits) {
        case 1: return launch_decode_s<D, 1>(p, s);
        case 2: return launch_decode_s<D, 2>(p, s);
        case 4: return launch_decode_s<D, 4>(p, s);
        case 8: return launch_decode_s<D, 8>(p, s);
        default: return launch_decode_s<D, 16>(p, s);
    }
}

}  // namespace
}  // namespace ssa

using namespace ssa;

extern "C" size_t sparse_attn_decode_ws_bytes(int B, int H_q, int d) {
    if (B <= 0 || H_q <= 0 || d <= 0) return 0;
    return static_cast<size_t>(B) * H_q * dec_splits(B, H_q) * (2 + d) * sizeof(float);
}

extern "C" int sparse_attn_decode(const void *Q, const void *K, const void *V, int B, int H_q,
                                  int H_kv, int S_cache, int d, const int32_t *pos,
                                  const ssa_plan *plan, const int32_t *kv_map, float scale,
                                  void *O, float *LSE, void *ws, size_t ws_bytes,
                                  int32_t *dev_status, void *stream) {
    ssa::TraceRange trace_range("sparse_attn_decode");
    SSA_CHECK_ARG(Q && K && V && pos && plan && O && LSE && ws,
                  "sparse_attn_decode: null pointer argument");
    if (d != 64 && d != 128) {
        set_error("sparse_attn_decode: head dimension must be 64 or 128 (got %d)", d);
        return SSA_ERR_UNSUPPORTED;
    }
    SSA_CHECK_ARG(B >= 1 && H_q >= 1 && H_kv >= 1 && S_cache >= 1,
                  "sparse_attn_decode: B, H_q, H_kv, S_cache must be >= 1");
    SSA_CHECK_ARG(B <= 65535 && H_q <= 65535, "sparse_attn_decode: B and H_q must be <= 65535");
    SSA_CHECK_ARG(kv_map || H_q % H_kv == 0,
                  "sparse_attn_decode: H_q (%d) must be a multiple of H_kv (%d) without kv_map", H_q,
                  H_kv);
    if (plan->bitmap_slots != 0) {
        set_error("sparse_attn_decode: Case-2 plans (element-bitmap tiles) are not supported by decoding");
        return SSA_ERR_UNSUPPORTED;
    }
    SSA_CHECK_ARG(plan->S == S_cache && plan->n_heads == H_q,
                  "sparse_attn_decode: plan (S=%d heads=%d) does not match S_cache=%d H_q=%d", plan->S,
                  plan->n_heads, S_cache, H_q);
    SSA_CHECK_ARG(plan->ext_diag_ptr && plan->ext_diag_offsets && plan->ext_vert_ptr && plan->ext_vert_cols,
                  "sparse_attn_decode: null plan list");
    SSA_CHECK_ARG(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O) && aligned16(ws),
                  "sparse_attn_decode: Q, K, V, O and ws must be 16-byte aligned");
    SSA_CHECK_ARG(scale > 0.0f && scale < 1e30f, "sparse_attn_decode: scale must be positive and finite");
    const size_t need = sparse_attn_decode_ws_bytes(B, H_q, d);
    if (ws_bytes < need) {
        set_error("sparse_attn_decode: workspace %zu bytes < required %zu", ws_bytes, need);
        return SSA_ERR_CAPACITY;
    }
    DecParams p{};
    p.B = B;
    p.H = H_q;
    p.Hkv = H_kv;
    p.S = S_cache;
    p.d = d;
    p.splits = dec_splits(B, H_q);
    p.Q = static_cast<const uint16_t *>(Q);
    p.K = static_cast<const uint16_t *>(K);
    p.V = static_cast<const uint16_t *>(V);
    p.pos = pos;
    p.dptr = plan->ext_diag_ptr;
    p.doff = plan->ext_diag_offsets;
    p.vptr = plan->ext_vert_ptr;
    p.vcol = plan->ext_vert_cols;
    p.kv_map = kv_map;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.part = static_cast<float *>(ws);
    p.O = static_cast<uint16_t *>(O);
    p.LSE = LSE;
    p.status = dev_status;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d == 64 ? launch_decode<64>(p, s) : launch_decode<128>(p, s);
}
