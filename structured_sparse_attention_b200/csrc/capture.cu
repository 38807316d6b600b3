// capture.cu -- stage one of DAM on the GPU: Box-Cox, row scaling, threshold, gamma
// scoring and selection (DAM review page, "What carries the argument"; lambda, tau,
// mu from "Assumptions & free parameters"; eps from Referee Report minor comment 1).
//
// Kernels
//   capture_hits_kernel    one pass over the causal half of every map: per row the
//                          min/max, the exact float32 cut point x* of the decision
//                          t(x) >= tau, and the hit counts of every diagonal and column
//   capture_select_kernel  gamma = hits / cells in fp64, keep gamma >= mu, ordered
//                          compaction per map
//   capture_pack_kernel    CSR offsets across maps and the final lists
//
// Exactness.  The decision for an entry x is made by the sequence
//   z = x + eps; s = sqrt(z); y = (s - 1) / lambda; t = (y - y_lo) / (y_hi - y_lo); t >= tau
// in correctly rounded fp64 (lambda = 1 drops the sqrt), with y_lo / y_hi the same
// sequence at the row min / max.  Every step is monotone non-decreasing in x, so for
// the non-negative floats of a row there is one cut point x* with
// decision(x) == (x >= x*).  The kernel finds x* exactly by evaluating the very same
// sequence on candidate floats (a window around the closed-form estimate, then a
// 33-way bracketing search), so each decision equals the one obtained by evaluating
// the sequence at every entry.  Each row thus costs a few fp64 evaluations per lane
// instead of one per entry.
#include <type_traits>

#include "common.cuh"

namespace ssa {
namespace {

constexpr int kCaptureThreads = 256;
constexpr int kCaptureWarps = kCaptureThreads / 32;

struct CaptureParams {
    const float *maps;
    int n_maps;
    int L;
    double lambda;
    double tau;
    double mu;
    double eps;
    int32_t *hits;     // [n_maps][2][L]
    int32_t *staging;  // [n_maps][2][L]
    int32_t *counts;   // [n_maps][2]
    int32_t *diag_ptr;
    int32_t *diag_offsets;
    int32_t *vert_ptr;
    int32_t *vert_cols;
    int32_t *status;
    int row_chunks;  // CTAs per map of the hits kernel; rows interleaved across them
    int scaling;     // 0: min and max of each row's causal entries; 1: of the whole map's
    uint32_t *map_mm;  // per map: min and max bits of its causal entries (scaling 1)
    uint32_t *bits;    // optional true mask [n_maps][L][bits_words] (bit j of row i), or null
    int bits_words;    // ceil(L / 32)
};

// Box-Cox of x + eps: ((x + eps)^lambda - 1) / lambda, log(x + eps) at lambda = 0.  At
// lambda 1/2 and 1 every step is correctly rounded (sqrt, +, -, /), as in the oracle;
// other lambdas use pow / log, which are not correctly rounded on either side, so a
// decision within a few units in the last place of tau may differ from the oracle's.
// Transform kinds: TR_SQRT (lambda = 1/2), TR_LINEAR (lambda = 1), TR_POW (any other).
constexpr int TR_SQRT = 0, TR_LINEAR = 1, TR_POW = 2;

template <int TR>
__device__ __forceinline__ double box_cox_rn(double x, double eps, double lambda) {
    double z = __dadd_rn(x, eps);
    if constexpr (TR == TR_SQRT) return __ddiv_rn(__dsub_rn(__dsqrt_rn(z), 1.0), lambda);
    if constexpr (TR == TR_LINEAR) return __ddiv_rn(__dsub_rn(z, 1.0), lambda);
    if (lambda == 0.0) return log(z);
    return __ddiv_rn(__dsub_rn(pow(z, lambda), 1.0), lambda);
}

template <int TR>
__device__ __forceinline__ bool decide(uint32_t xbits, double eps, double lambda, double ylo, double yrange,
                                       double tau) {
    double x = static_cast<double>(__uint_as_float(xbits));
    double t = __ddiv_rn(__dsub_rn(box_cox_rn<TR>(x, eps, lambda), ylo), yrange);
    return t >= tau;
}

// Smallest float bit pattern u in [u0, u1] with decide(u) true, or u1 + 1 if none.
// Collective over the warp; every lane returns the same value.
template <int TR>
__device__ uint32_t find_cut(uint32_t u0, uint32_t u1, float mn, float mx, double eps, double lambda,
                             double tau) {
    const int lane = threadIdx.x & 31;
    const double ylo = box_cox_rn<TR>(static_cast<double>(mn), eps, lambda);
    const double yhi = box_cox_rn<TR>(static_cast<double>(mx), eps, lambda);
    const double yrange = __dsub_rn(yhi, ylo);
    // Closed-form estimate of the cut (only steers the first probe window).
    double est;
    if constexpr (TR == TR_SQRT) {
        double a = sqrt(static_cast<double>(mn) + eps), b = sqrt(static_cast<double>(mx) + eps);
        double s = a + tau * (b - a);
        est = s * s - eps;
    } else if constexpr (TR == TR_LINEAR) {
        est = static_cast<double>(mn) + tau * (static_cast<double>(mx) - static_cast<double>(mn));
    } else if (lambda == 0.0) {
        const double a = log(static_cast<double>(mn) + eps), b = log(static_cast<double>(mx) + eps);
        est = exp(a + tau * (b - a)) - eps;
    } else {
        const double a = pow(static_cast<double>(mn) + eps, lambda), b = pow(static_cast<double>(mx) + eps, lambda);
        est = pow(a + tau * (b - a), 1.0 / lambda) - eps;
    }
    float ef = static_cast<float>(est);
    if (!(ef >= mn)) ef = mn;
    if (!(ef <= mx)) ef = mx;
    const int64_t ue = static_cast<int64_t>(__float_as_uint(ef));

    int64_t lo = static_cast<int64_t>(u0) - 1;  // decide(lo) == false (virtual below u0)
    int64_t hi = static_cast<int64_t>(u1) + 1;  // decide(hi) == true  (virtual above u1)
    for (int round = 0; round < 24 && hi - lo > 1; ++round) {
        const int64_t inside = hi - lo - 1;
        int64_t first, step_num = 0;
        int np;
        bool window = false;
        if (round == 0) {
            first = ue - 16;
            if (first < lo + 1) first = lo + 1;
            int64_t last = first + 31;
            if (last > hi - 1) last = hi - 1;
            np = static_cast<int>(last - first + 1);
            window = true;
        } else if (inside <= 32) {
            first = lo + 1;
            np = static_cast<int>(inside);
            window = true;
        } else {
            first = lo;
            step_num = hi - lo;
            np = 32;
        }
        int64_t p = window ? first + lane : first + (step_num * (lane + 1)) / 33;
        bool val = true;
        if (lane < np) val = decide<TR>(static_cast<uint32_t>(p), eps, lambda, ylo, yrange, tau);
        const uint32_t ball = __ballot_sync(0xffffffffu, val);
        // first true (lanes >= np report true); 32 when all 32 probes are false
        const int f = ball ? (__ffs(ball) - 1) : 32;
        const int64_t pf = __shfl_sync(0xffffffffu, p, f < 31 ? f : 31);
        const int64_t pprev = __shfl_sync(0xffffffffu, p, f > 0 ? f - 1 : 0);
        if (f < np) hi = pf;
        if (f > 0) lo = pprev;
    }
    return static_cast<uint32_t>(hi);
}

template <int MAXK, int TR>
__global__ void __launch_bounds__(kCaptureThreads)
    capture_hits_kernel(CaptureParams p) {
    extern __shared__ int32_t s_hist[];  // [2][L]: diagonal hits, column hits
    const int L = p.L;
    const int m = blockIdx.x / p.row_chunks;
    const int chunk = blockIdx.x % p.row_chunks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int k = threadIdx.x; k < 2 * L; k += kCaptureThreads) s_hist[k] = 0;
    __syncthreads();

    const float *map = p.maps + static_cast<size_t>(m) * L * L;
    bool bad = false;
    // per-map scaling: one cut for the whole map, from its min and max (found by warp 0)
    __shared__ uint32_t s_map_cut;
    if (p.scaling == 1) {
        if (warp == 0) {
            const float mn = __uint_as_float(p.map_mm[2 * m]), mx = __uint_as_float(p.map_mm[2 * m + 1]);
            const uint32_t u0 = __float_as_uint(mn), u1 = __float_as_uint(mx);
            const uint32_t c = (u0 == u1) ? ((1.0 >= p.tau) ? 0u : 0xffffffffu)
                                          : find_cut<TR>(u0, u1, mn, mx, p.eps, p.lambda, p.tau);
            if (lane == 0) s_map_cut = c;
        }
        __syncthreads();
    }
    // Rows are software-pipelined: the loads of the warp's next row are issued before the
    // current row's cut point is searched, so each warp keeps a row in flight while it
    // computes (the search is a chain of dependent fp64 steps).
    auto load_row = [&](int i, float (&x)[MAXK]) {
        const float *row = map + static_cast<size_t>(i) * L;
#pragma unroll
        for (int k = 0; k < MAXK; ++k) {
            const int j = lane + 32 * k;
            x[k] = (i < L && j <= i) ? __ldg(row + j) : 0.0f;
        }
    };
    const int stride = p.row_chunks * kCaptureWarps;
    int i = chunk + p.row_chunks * warp;
    float xc[MAXK], xn[MAXK];
    load_row(i, xc);
    for (; i < L; i += stride) {
        load_row(i + stride, xn);
        const int n = i + 1;
        float mn = __int_as_float(0x7f800000), mx = 0.0f;
#pragma unroll
        for (int k = 0; k < MAXK; ++k) {
            const int j = lane + 32 * k;
            if (j < n) {
                float x = xc[k];
                if (!(x >= 0.0f) || x == __int_as_float(0x7f800000)) bad = true;
                if (__float_as_uint(x) == 0x80000000u) x = 0.0f;  // -0 counts as +0
                xc[k] = x;
                mn = fminf(mn, x);
                mx = fmaxf(mx, x);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        uint32_t cut;
        const uint32_t u0 = __float_as_uint(mn), u1 = __float_as_uint(mx);
        if (p.scaling == 1) {
            cut = s_map_cut;
        } else if (u0 == u1) {
            cut = (1.0 >= p.tau) ? 0u : 0xffffffffu;  // constant row: t = 1
        } else {
            cut = find_cut<TR>(u0, u1, mn, mx, p.eps, p.lambda, p.tau);
        }
        // for non-negative floats the order of the values is the order of their bits, so
        // x >= x* is the comparison of the bit patterns (a cut of 0xffffffff keeps none)
#pragma unroll
        for (int k = 0; k < MAXK; ++k) {
            const int j = lane + 32 * k;
            const bool on = j < n && __float_as_uint(xc[k]) >= cut;
            if (on) {
                atomicAdd(&s_hist[i - j], 1);
                atomicAdd(&s_hist[L + j], 1);
            }
            if (p.bits) {
                // the row's true mask, 32 columns per word
                const uint32_t word = __ballot_sync(0xffffffffu, on);
                if (lane == 0 && k < p.bits_words)
                    p.bits[(static_cast<size_t>(m) * L + i) * p.bits_words + k] = word;
            }
        }
#pragma unroll
        for (int k = 0; k < MAXK; ++k) xc[k] = xn[k];
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) report(p.status, SSA_ERR_INVALID);
    __syncthreads();
    int32_t *hits = p.hits + static_cast<size_t>(m) * 2 * L;
    for (int k = threadIdx.x; k < 2 * L; k += kCaptureThreads) {
        const int v = s_hist[k];
        if (v) atomicAdd(hits + k, v);
    }
}

// Multiprocessors of the current device (cached per device).
int sm_count_capture() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// Per-map min and max of the causal entries (scaling 1), as float bit patterns: for the
// non-negative floats of a map the order of the bits is the order of the values (-0 is
// taken as +0).  map_mm must hold {0xffffffff, 0} per map on entry.
__global__ void __launch_bounds__(kCaptureThreads) capture_minmax_kernel(CaptureParams p) {
    const int L = p.L;
    const int m = blockIdx.x / p.row_chunks;
    const int chunk = blockIdx.x % p.row_chunks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *map = p.maps + static_cast<size_t>(m) * L * L;
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (int i = chunk + p.row_chunks * warp; i < L; i += p.row_chunks * kCaptureWarps) {
        const float *row = map + static_cast<size_t>(i) * L;
        for (int j = lane; j <= i; j += 32) {
            uint32_t b = __float_as_uint(__ldg(row + j));
            if (b == 0x80000000u) b = 0;
            mn = min(mn, b);
            mx = max(mx, b);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
        atomicMin(p.map_mm + 2 * m, mn);
        atomicMax(p.map_mm + 2 * m + 1, mx);
    }
}

// {0xffffffff, 0} for every map: the identities of the min / max reductions.
__global__ void capture_minmax_init_kernel(uint32_t *mm, int n_maps) {
    const int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m < n_maps) {
        mm[2 * m] = 0xffffffffu;
        mm[2 * m + 1] = 0u;
    }
}

// Ordered compaction of {x in [0, L) : keep(x)} by the whole block.
template <typename Pred>
__device__ int block_compact(int L, Pred keep, int32_t *out, int32_t *s_warp) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int base = 0;
    for (int start = 0; start < L; start += kCaptureThreads) {
        const int x = start + threadIdx.x;
        const bool k = (x < L) && keep(x);
        const uint32_t ball = __ballot_sync(0xffffffffu, k);
        if (lane == 0) s_warp[warp] = __popc(ball);
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < kCaptureWarps; ++w) {
            const int c = s_warp[w];
            if (w < warp) before += c;
            total += c;
        }
        if (k) out[base + before + __popc(ball & ((1u << lane) - 1u))] = x;
        base += total;
        __syncthreads();
    }
    return base;
}

__global__ void __launch_bounds__(kCaptureThreads) capture_select_kernel(CaptureParams p) {
    __shared__ int32_t s_warp[kCaptureWarps];
    const int L = p.L;
    const int m = blockIdx.x;
    const int32_t *hd = p.hits + static_cast<size_t>(m) * 2 * L;
    const int32_t *hc = hd + L;
    int32_t *sd = p.staging + static_cast<size_t>(m) * 2 * L;
    int32_t *sc = sd + L;
    const double mu = p.mu;
    // gamma_k = sum(M P_k) / sum(P_k): pattern r (or c) has L - r (L - c) cells.
    const int nd = block_compact(
        L,
        [&](int r) {
            return __ddiv_rn(static_cast<double>(hd[r]), static_cast<double>(L - r)) >= mu;
        },
        sd, s_warp);
    const int nc = block_compact(
        L,
        [&](int c) {
            return __ddiv_rn(static_cast<double>(hc[c]), static_cast<double>(L - c)) >= mu;
        },
        sc, s_warp);
    if (threadIdx.x == 0) {
        p.counts[2 * m] = nd;
        p.counts[2 * m + 1] = nc;
    }
}

__global__ void __launch_bounds__(kCaptureThreads) capture_pack_kernel(CaptureParams p) {
    __shared__ int32_t s_red[2][kCaptureWarps];
    const int L = p.L;
    const int m = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int od = 0, oc = 0;
    for (int q = threadIdx.x; q < m; q += kCaptureThreads) {
        od += p.counts[2 * q];
        oc += p.counts[2 * q + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        od += __shfl_xor_sync(0xffffffffu, od, o);
        oc += __shfl_xor_sync(0xffffffffu, oc, o);
    }
    if (lane == 0) {
        s_red[0][warp] = od;
        s_red[1][warp] = oc;
    }
    __syncthreads();
    od = oc = 0;
    for (int w = 0; w < kCaptureWarps; ++w) {
        od += s_red[0][w];
        oc += s_red[1][w];
    }
    const int nd = p.counts[2 * m], nc = p.counts[2 * m + 1];
    const int32_t *sd = p.staging + static_cast<size_t>(m) * 2 * L;
    const int32_t *sc = sd + L;
    for (int k = threadIdx.x; k < nd; k += kCaptureThreads) p.diag_offsets[od + k] = sd[k];
    for (int k = threadIdx.x; k < nc; k += kCaptureThreads) p.vert_cols[oc + k] = sc[k];
    if (threadIdx.x == 0) {
        p.diag_ptr[m] = od;
        p.vert_ptr[m] = oc;
        if (m == p.n_maps - 1) {
            p.diag_ptr[m + 1] = od + nd;
            p.vert_ptr[m + 1] = oc + nc;
        }
    }
}

}  // namespace
}  // namespace ssa

using namespace ssa;

extern "C" size_t sparse_pattern_capture_ws_bytes(int n_maps, int L) {
    if (n_maps <= 0 || L <= 0) return 0;
    return static_cast<size_t>(n_maps) * (4 * static_cast<size_t>(L) + 2) * sizeof(int32_t);
}

extern "C" int sparse_pattern_capture_ex(const float *maps, int n_maps, int L, double lambda,
                                         double tau, double mu, double eps, int scaling,
                                         int32_t *diag_ptr, int32_t *diag_offsets,
                                         int32_t *vert_ptr, int32_t *vert_cols,
                                         uint32_t *true_mask, void *ws, size_t ws_bytes,
                                         int32_t *dev_status, void *stream) {
    SSA_CHECK_ARG(maps && diag_ptr && diag_offsets && vert_ptr && vert_cols && ws,
                  "sparse_pattern_capture: null pointer argument");
    SSA_CHECK_ARG(n_maps >= 1, "sparse_pattern_capture: n_maps must be >= 1 (got %d)", n_maps);
    if (L < 1 || L > 1024) {
        set_error("sparse_pattern_capture: L must be in [1, 1024] (got %d)", L);
        return L < 1 ? SSA_ERR_INVALID : SSA_ERR_UNSUPPORTED;
    }
    SSA_CHECK_ARG(lambda >= 0.0 && lambda <= 64.0, "sparse_pattern_capture: lambda must be in [0, 64] (got %g)",
                  lambda);
    SSA_CHECK_ARG(scaling == SSA_SCALE_ROW || scaling == SSA_SCALE_MAP,
                  "sparse_pattern_capture: scaling must be SSA_SCALE_ROW or SSA_SCALE_MAP (got %d)", scaling);
    SSA_CHECK_ARG((reinterpret_cast<uintptr_t>(true_mask) & 3u) == 0,
                  "sparse_pattern_capture: true_mask must be 4-byte aligned");
    SSA_CHECK_ARG(eps >= 0.0 && eps < 1e300, "sparse_pattern_capture: eps must be finite and >= 0");
    SSA_CHECK_ARG(tau == tau && mu == mu, "sparse_pattern_capture: tau and mu must not be NaN");
    SSA_CHECK_ARG((reinterpret_cast<uintptr_t>(ws) & 3u) == 0,
                  "sparse_pattern_capture: ws must be 4-byte aligned");
    SSA_CHECK_ARG(static_cast<size_t>(n_maps) * L * L < (static_cast<size_t>(1) << 40),
                  "sparse_pattern_capture: maps too large");
    const size_t need = sparse_pattern_capture_ws_bytes(n_maps, L);
    if (ws_bytes < need) {
        set_error("sparse_pattern_capture: workspace %zu bytes < required %zu", ws_bytes, need);
        return SSA_ERR_CAPACITY;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CaptureParams p;
    p.maps = maps;
    p.n_maps = n_maps;
    p.L = L;
    p.lambda = lambda;
    p.tau = tau;
    p.mu = mu;
    p.eps = eps;
    p.hits = static_cast<int32_t *>(ws);
    p.staging = p.hits + static_cast<size_t>(n_maps) * 2 * L;
    p.counts = p.staging + static_cast<size_t>(n_maps) * 2 * L;
    p.diag_ptr = diag_ptr;
    p.diag_offsets = diag_offsets;
    p.vert_ptr = vert_ptr;
    p.vert_cols = vert_cols;
    p.status = dev_status;
    p.scaling = scaling;
    p.map_mm = reinterpret_cast<uint32_t *>(p.staging);  // free until the select kernel
    p.bits = true_mask;
    p.bits_words = (L + 31) / 32;

    SSA_CUDA_TRY(cudaMemsetAsync(p.hits, 0, static_cast<size_t>(n_maps) * 2 * L * sizeof(int32_t), s));
    const size_t smem = 2 * static_cast<size_t>(L) * sizeof(int32_t);
    // Enough CTAs to fill the GPU a few times over even for a few maps (each warp then
    // takes fewer rows), at most one row per warp.
    int chunks = 8;
    while (chunks < 64 && static_cast<long long>(n_maps) * chunks < 4LL * sm_count_capture() &&
           chunks * 2 * kCaptureWarps <= L)
        chunks *= 2;
    p.row_chunks = chunks;
    const unsigned grid = static_cast<unsigned>(n_maps) * chunks;
    if (scaling == SSA_SCALE_MAP) {
        capture_minmax_init_kernel<<<(n_maps + 255) / 256, 256, 0, s>>>(p.map_mm, n_maps);
        SSA_LAUNCH_CHECK();
        capture_minmax_kernel<<<grid, kCaptureThreads, 0, s>>>(p);
        SSA_LAUNCH_CHECK();
    }
    const int tr = lambda == 0.5 ? TR_SQRT : (lambda == 1.0 ? TR_LINEAR : TR_POW);
    auto launch_hits = [&](auto MK) {
        constexpr int MAXK = decltype(MK)::value;
        if (tr == TR_SQRT) capture_hits_kernel<MAXK, TR_SQRT><<<grid, kCaptureThreads, smem, s>>>(p);
        else if (tr == TR_LINEAR) capture_hits_kernel<MAXK, TR_LINEAR><<<grid, kCaptureThreads, smem, s>>>(p);
        else capture_hits_kernel<MAXK, TR_POW><<<grid, kCaptureThreads, smem, s>>>(p);
    };
    if (L <= 512) launch_hits(std::integral_constant<int, 16>{});
    else launch_hits(std::integral_constant<int, 32>{});
    SSA_LAUNCH_CHECK();
    capture_select_kernel<<<n_maps, kCaptureThreads, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    capture_pack_kernel<<<n_maps, kCaptureThreads, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    return SSA_OK;
}

extern "C" int sparse_pattern_capture(const float *maps, int n_maps, int L, double lambda,
                                      double tau, double mu, double eps, int32_t *diag_ptr,
                                      int32_t *diag_offsets, int32_t *vert_ptr,
                                      int32_t *vert_cols, void *ws, size_t ws_bytes,
                                      int32_t *dev_status, void *stream) {
    return sparse_pattern_capture_ex(maps, n_maps, L, lambda, tau, mu, eps, SSA_SCALE_ROW, diag_ptr,
                                     diag_offsets, vert_ptr, vert_cols, nullptr, ws, ws_bytes,
                                     dev_status, stream);
}

// ---------------------------------------------------------------------------------
// Allocation-free variant of sparse_pattern_capture.
//
// Its scratch (hit counts, staging lists and per-map counts) lives in a file-scope
// device array instead of a caller-provided workspace.  Every GPU that loads the
// library holds this array until the process exits.  All calls share it and it
// keeps the last call's contents: the call clears the hit counts itself (the only
// part that must start at zero), and calls whose work overlaps on the GPU (other
// streams, other host threads) race on it.
// ---------------------------------------------------------------------------------
#include <mutex>

namespace ssa {

constexpr size_t kNoAllocScratchBytes = SSA_CAPTURE_NOALLOC_SCRATCH_BYTES;

// The scratch itself: a file-scope static device array (internal linkage).
static __device__ __align__(256) int32_t g_capture_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

namespace {

constexpr int kMaxDevices = 64;

std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_capture_scratch on the current device.  Looked up once per
// device, with that device current; in host code the array's name is only a host-side
// stand-in, never a device address.
int scratch_address(void **out) {
    int dev = -1;
    SSA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) {
        set_error("sparse_pattern_capture_noalloc: device ordinal %d out of range", dev);
        return SSA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        SSA_CUDA_TRY(cudaGetSymbolAddress(&p, g_capture_scratch));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SSA_OK;
}

}  // namespace
}  // namespace ssa

extern "C" int sparse_pattern_capture_noalloc(const float *maps, int n_maps, int L, double lambda,
                                              double tau, double mu, double eps, int32_t *diag_ptr,
                                              int32_t *diag_offsets, int32_t *vert_ptr,
                                              int32_t *vert_cols, int32_t *dev_status,
                                              void *stream) {
    SSA_CHECK_ARG(n_maps >= 1 && L >= 1, "sparse_pattern_capture_noalloc: n_maps and L must be >= 1");
    const size_t need = sparse_pattern_capture_ws_bytes(n_maps, L);
    if (need > kNoAllocScratchBytes) {
        set_error("sparse_pattern_capture_noalloc: %d maps of %d x %d need %zu scratch bytes, more "
                  "than the fixed %zu; use sparse_pattern_capture with a workspace",
                  n_maps, L, L, need, kNoAllocScratchBytes);
        return SSA_ERR_CAPACITY;
    }
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != SSA_OK) return rc;
    return sparse_pattern_capture(maps, n_maps, L, lambda, tau, mu, eps, diag_ptr, diag_offsets,
                                  vert_ptr, vert_cols, scratch, kNoAllocScratchBytes, dev_status,
                                  stream);
}
