// maps.cu -- stage one, step 1: averaged causal attention maps at capture length L.
//
// Stage one of DAM starts from attention maps averaged over a calibration corpus at
// L = 512 (DAM review page: "What carries the argument"; "Assumptions & free
// parameters").  This kernel produces them on the GPU from B samples of per-head Q, K:
//   maps[m][i][j] = (1/B) sum_b softmax_j(scale * Q[m][b][i] . K[m][b][j])   (j <= i)
//   maps[m][i][j] = 0                                                        (j > i)
// in the layout sparse_pattern_capture reads.
//
// One CTA per (map, 128-row block rb); the row block's keys are the chunks c = 0..rb of
// 128 keys, and a tile is one 128 x 128 block S = Q_b K_(b,c)^T (tcgen05, fp32 in TMEM):
//   pass 1 (samples outer, chunks inner): per row the running max and sum of 2^(x - max)
//          over the causal keys of sample b  ->  (m_b, 1 / l_b) kept in shared memory
//   pass 2 (chunks outer, samples inner): the same tiles again; P = 2^(x - m_b) / l_b
//          accumulated in registers over the samples, then the chunk of the map row is
//          written once.
// Each exponential is taken twice (once per pass): accumulating a whole row block over
// all its chunks at once would need (rb + 1) x 128 fp32 values per row.
//
// Roles (320 threads): warps 0-7 softmax, two warpgroups splitting each tile's columns
// (warpgroup h takes columns 64h..64h+63; thread il of a warpgroup owns row 128 rb + il,
// TMEM lane il), so two warps per SM sub-partition share the MUFU; the halves' running
// max and sum are combined through shared memory at the end of each sample.  Warp 8
// lane 0: TMA producer of the Q block and K chunk of each tile.  Warp 9: tensor memory
// (two S buffers of 128 columns) and lane 0 issues the MMAs.
//
// Every wait is bounded: on expiry the kernel records SSA_ERR_TIMEOUT, stops every role,
// drains its copies and MMAs, frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace ssa {
namespace {

constexpr int kMapsMaxB = SSA_MAPS_MAX_B;
constexpr int kMThreads = 320;
constexpr int kMSoftmaxThreads = 256;
constexpr int kMWarpTma = 8, kMWarpMma = 9;
constexpr uint32_t kMTmemCols = 256;
constexpr int kMBoxBytes = 128 * 128;  // 128 rows x 64 bf16, one 128-byte swizzle span
constexpr int64_t kMDrainNs = 1000000000LL;

template <int D>
struct MCfg {
    static constexpr int NS = (D == 64) ? 4 : 2;        // smem stages (Q block + K chunk)
    static constexpr int BOXES = D / 64;
    static constexpr int TILE = BOXES * kMBoxBytes;     // one 128-row bf16 operand
    static constexpr int STAGE = 2 * TILE;
    static constexpr int OFF_STAT = NS * STAGE;         // float2 [2 halves][MAXB][128]
    static constexpr int OFF_XCH = OFF_STAT + 2 * kMapsMaxB * 128 * 8;  // float2 [2][2][128]
    static constexpr int OFF_BAR = OFF_XCH + 2 * 2 * 128 * 8;
    static constexpr int SMEM = OFF_BAR + 1024 + 1024;  // barrier block + alignment slack
    static_assert(SMEM <= 232448, "shared memory budget exceeded");
};

struct MShared {
    uint64_t full[4], empty[4];
    uint64_t s_full[2], s_empty[2];
    uint64_t xch[2];
    uint64_t mma_drain, sm_done;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(MShared) <= 1024, "barrier block too large");

struct MapsParams {
    int n_maps, B, L, nrb;
    float scale_log2, inv_B;
    float *maps;
    int32_t *status;
    int64_t wait_ns;
    int align32;  // maps is 32-byte aligned (rows are then too: L * 4 is a multiple of 512)
};

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 "version 1" format).
__device__ __forceinline__ uint64_t m_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 A/B, fp32 accumulate, A and B K-major.
__host__ __device__ constexpr uint32_t m_idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// Tile t of the CTA's sequence: pass 1 for t < nc B (b = t / nc, c = t % nc), then
// pass 2 (c = t' / B, b = t' % B).
__device__ __forceinline__ void m_tile(int t, int nc, int B, bool &pass2, int &b, int &c) {
    const int n1 = nc * B;
    pass2 = t >= n1;
    if (!pass2) {
        b = t / nc;
        c = t - b * nc;
    } else {
        const int u = t - n1;
        c = u / B;
        b = u - c * B;
    }
}

template <int D>
__global__ void __launch_bounds__(kMThreads, 1)
    attn_maps_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const MapsParams p) {
    using C = MCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    MShared *sh = reinterpret_cast<MShared *>(smem + C::OFF_BAR);
    volatile int *abort = &sh->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // larger row blocks (more chunks) first
    const int rb = p.nrb - 1 - static_cast<int>(blockIdx.x) / p.n_maps;
    const int map = static_cast<int>(blockIdx.x) % p.n_maps;
    const int nc = rb + 1;
    const int T = 2 * nc * p.B;
    const int64_t lim = p.wait_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh->s_full[s], 1);
            mbar_init(&sh->s_empty[s], kMSoftmaxThreads);
            mbar_init(&sh->xch[s], kMSoftmaxThreads);
        }
        mbar_init(&sh->mma_drain, 1);
        mbar_init(&sh->sm_done, kMSoftmaxThreads);
        sh->abort = 0;
        fence_barrier_init();
    }
    if (warp == kMWarpMma) {
        tmem_alloc(&sh->tmem_base, kMTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;

    if (warp == kMWarpTma) {
        if (lane == 0) {
            // ------------------------------ TMA producer ------------------------------
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            bool ok = true;
            int t = 0;
            for (; t < T; ++t) {
                const int st = t % C::NS;
                if (t >= C::NS && !mbar_wait(&sh->empty[st], ((t / C::NS) - 1) & 1, lim, abort)) {
                    ok = false;
                    break;
                }
                bool pass2;
                int b, c;
                m_tile(t, nc, p.B, pass2, b, c);
                const int z = map * p.B + b;
                uint8_t *dq = smem + st * C::STAGE;
                mbar_arrive_expect_tx(&sh->full[st], C::STAGE);
                for (int x = 0; x < C::BOXES; ++x) {
                    tma_load_3d(dq + x * kMBoxBytes, &tmQ, &sh->full[st], 64 * x, 128 * rb, z);
                    tma_load_3d(dq + C::TILE + x * kMBoxBytes, &tmK, &sh->full[st], 64 * x, 128 * c, z);
                }
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            // never leave the CTA with a copy still writing shared memory
            for (int u = (t > C::NS ? t - C::NS : 0); u < t; ++u)
                mbar_wait(&sh->full[u % C::NS], (u / C::NS) & 1, kMDrainNs, nullptr);
        }
    } else if (warp == kMWarpMma) {
        if (lane == 0) {
            // ------------------------------- MMA issuer -------------------------------
            constexpr uint32_t IDESC = m_idesc(128, 128);
            bool ok = true;
            for (int t = 0; t < T && ok; ++t) {
                const int st = t % C::NS, sb = t & 1;
                if (!mbar_wait(&sh->full[st], (t / C::NS) & 1, lim, abort)) ok = false;
                if (ok && t >= 2 && !mbar_wait(&sh->s_empty[sb], ((t >> 1) - 1) & 1, lim, abort)) ok = false;
                if (!ok) break;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + st * C::STAGE);
                const uint32_t sK = sQ + C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // A = Q block, B = K chunk, both K-major: 16 elements = 32 B per step
                    const uint32_t off = (kk >> 2) * kMBoxBytes + (kk & 3) * 32;
                    umma_ss(tmem + 128 * sb, m_sdesc(sQ + off, 16, 1024), m_sdesc(sK + off, 16, 1024), IDESC,
                            kk > 0 ? 1u : 0u);
                }
                umma_commit(&sh->s_full[sb]);
                umma_commit(&sh->empty[st]);
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            umma_commit(&sh->mma_drain);
        }
        __syncwarp();
        if (lane == 0) {
            mbar_wait(&sh->sm_done, 0, kMDrainNs, nullptr);
            mbar_wait(&sh->mma_drain, 0, kMDrainNs, nullptr);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kMTmemCols);
    } else {
        // --------------------------------- softmax ---------------------------------
        const int h = warp >> 2;  // column half of every tile
        const int il = 32 * (warp & 3) + lane;
        const int i = 128 * rb + il;
        const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        float2 *stat = reinterpret_cast<float2 *>(smem + C::OFF_STAT) + h * kMapsMaxB * 128;
        float2 *xch = reinterpret_cast<float2 *>(smem + C::OFF_XCH);  // [parity][half][row]
        const float sl2 = p.scale_log2;
        float *row = p.maps + (static_cast<size_t>(map) * p.L + i) * p.L;
        bool ok = true;
        float m = -INFINITY, l = 0.0f;
        float acc[64];
#pragma unroll
        for (int k = 0; k < 64; ++k) acc[k] = 0.0f;
        for (int t = 0; t < T; ++t) {
            bool pass2;
            int b, c;
            m_tile(t, nc, p.B, pass2, b, c);
            const int sb = t & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sh->s_full[sb], (t >> 1) & 1, lim, abort))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t r[64];
            const uint32_t tS = tmem + lane_off + 128 * sb + 64 * h;
            tmem_ld32(tS, r);
            tmem_ld32(tS + 32, r + 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sh->s_empty[sb]);  // the S buffer may take tile t + 2
            // causal keys of this row in the chunk: local column 64 h + k < nv
            const int nv = (c < rb) ? 128 : il + 1;
            const int kv = nv - 64 * h;  // k < kv active
            if (!pass2) {
                float x[64];
                float mx = -INFINITY;
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    x[k] = (k < kv) ? __uint_as_float(r[k]) * sl2 : -INFINITY;
                    mx = fmaxf(mx, x[k]);
                }
                const float m_new = fmaxf(m, mx);
                if (m_new != -INFINITY) {  // else no causal key in this half yet
                    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
                    for (int k = 0; k < 64; k += 4) {
                        s0 += ex2_approx(x[k] - m_new);
                        s1 += ex2_approx(x[k + 1] - m_new);
                        s2 += ex2_approx(x[k + 2] - m_new);
                        s3 += ex2_approx(x[k + 3] - m_new);
                    }
                    l = l * ex2_approx(m - m_new) + ((s0 + s1) + (s2 + s3));
                    m = m_new;
                }
                if (c == nc - 1) {
                    // combine the two halves of the row: both warpgroups compute the same
                    // (m_b, 1 / l_b) from the same two pairs
                    const int par = b & 1;
                    xch[(par * 2 + h) * 128 + il] = make_float2(m, l);
                    mbar_arrive(&sh->xch[par]);
                    if (!__all_sync(0xffffffffu, mbar_wait(&sh->xch[par], (b >> 1) & 1, lim, abort))) {
                        ok = false;
                        break;
                    }
                    const float2 o0 = xch[(par * 2 + 0) * 128 + il];
                    const float2 o1 = xch[(par * 2 + 1) * 128 + il];
                    const float mb = fmaxf(o0.x, o1.x);  // finite: key 0 is causal for every row
                    const float lb = o0.y * ex2_approx(o0.x - mb) + o1.y * ex2_approx(o1.x - mb);
                    stat[b * 128 + il] = make_float2(mb, 1.0f / lb);
                    m = -INFINITY;
                    l = 0.0f;
                }
            } else {
                const float2 st = stat[b * 128 + il];
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    const float e = ex2_approx(fmaf(__uint_as_float(r[k]), sl2, -st.x));
                    acc[k] = fmaf((k < kv) ? e : 0.0f, st.y, acc[k]);
                }
                if (b == p.B - 1) {
                    // the chunk of the map row, this half's 64 columns (256 bytes)
                    uint32_t w[64];
#pragma unroll
                    for (int k = 0; k < 64; ++k) {
                        w[k] = __float_as_uint(acc[k] * p.inv_B);
                        acc[k] = 0.0f;
                    }
                    float *dst = row + 128 * c + 64 * h;
                    if (p.align32) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) st_global_v8(dst + 8 * k, w + 8 * k);
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            reinterpret_cast<uint4 *>(dst)[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                    }
                }
            }
        }
        if (ok) {
            // the chunks above the diagonal block: zeros
            for (int cc = nc; cc < p.nrb; ++cc) {
                uint4 *dst = reinterpret_cast<uint4 *>(row + 128 * cc + 64 * h);
#pragma unroll
                for (int k = 0; k < 16; ++k) dst[k] = make_uint4(0, 0, 0, 0);
            }
        } else {
            report(p.status, SSA_ERR_TIMEOUT);
            *abort = 1;
        }
        tc_fence_before();
        mbar_arrive(&sh->sm_done);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 m_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 3-D map over bf16 [n_maps * B][L][d]; box = 64 columns x 128 rows x 1, 128-byte swizzle.
int m_make_map(CUtensorMap *m, const void *base, int d, int rows, int depth) {
    auto enc = m_encode_fn();
    if (!enc) {
        set_error("cuTensorMapEncodeTiled is unavailable");
        return SSA_ERR_CUDA;
    }
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(depth)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) for rows=%d depth=%d d=%d", static_cast<int>(r), rows,
                  depth, d);
        return SSA_ERR_CUDA;
    }
    return SSA_OK;
}

template <int D>
int launch_maps(const void *Q, const void *K, const MapsParams &p, cudaStream_t s) {
    using C = MCfg<D>;
    CUtensorMap mQ, mK;
    int rc;
    if ((rc = m_make_map(&mQ, Q, D, p.L, p.n_maps * p.B)) != SSA_OK) return rc;
    if ((rc = m_make_map(&mK, K, D, p.L, p.n_maps * p.B)) != SSA_OK) return rc;
    SSA_CUDA_TRY(cudaFuncSetAttribute(attn_maps_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    const unsigned grid = static_cast<unsigned>(p.n_maps) * static_cast<unsigned>(p.nrb);
    attn_maps_kernel<D><<<grid, kMThreads, C::SMEM, s>>>(mQ, mK, p);
    SSA_LAUNCH_CHECK();
    return SSA_OK;
}

}  // namespace
}  // namespace ssa

using namespace ssa;

extern "C" int sparse_attn_maps(const void *Q, const void *K, int n_maps, int B, int L, int d, float scale,
                                float *maps, int32_t *dev_status, void *stream) {
    SSA_CHECK_ARG(Q && K && maps, "sparse_attn_maps: null pointer argument");
    if (d != 64 && d != 128) {
        set_error("sparse_attn_maps: head dimension must be 64 or 128 (got %d)", d);
        return SSA_ERR_UNSUPPORTED;
    }
    SSA_CHECK_ARG(n_maps >= 1 && B >= 1 && B <= kMapsMaxB, "sparse_attn_maps: need n_maps >= 1 and 1 <= B <= %d",
                  kMapsMaxB);
    SSA_CHECK_ARG(L >= 128 && L <= SSA_MAPS_MAX_L && L % 128 == 0,
                  "sparse_attn_maps: L must be a multiple of 128 in [128, %d] (got %d)", SSA_MAPS_MAX_L, L);
    SSA_CHECK_ARG(static_cast<int64_t>(n_maps) * B < (1LL << 30) &&
                      static_cast<int64_t>(n_maps) * (L / 128) < (1LL << 31),
                  "sparse_attn_maps: too many maps");
    SSA_CHECK_ARG(aligned16(Q) && aligned16(K) && aligned16(maps),
                  "sparse_attn_maps: Q, K and maps must be 16-byte aligned");
    SSA_CHECK_ARG(scale > 0.0f && scale < 1e30f, "sparse_attn_maps: scale must be positive and finite");
    MapsParams p{};
    p.n_maps = n_maps;
    p.B = B;
    p.L = L;
    p.nrb = L / 128;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.inv_B = 1.0f / static_cast<float>(B);
    p.maps = maps;
    p.status = dev_status;
    p.wait_ns = wait_limit_ns();
    p.align32 = (reinterpret_cast<uintptr_t>(maps) & 31u) == 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d == 64 ? launch_maps<64>(Q, K, p, s) : launch_maps<128>(Q, K, p, s);
}
