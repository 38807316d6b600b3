// capture.cu -- stage one of DAM on the GPU: Box-Cox, row scaling, threshold, gamma
// scoring and selection (DAM review page, "What carries the argument"; lambda, tau,
// mu from "Assumptions & free parameters"; eps from Referee Report minor comment 1).
//
// Kernels
//   capture_minmax_kernel  (per-map scaling only) the min and max of every map's
//                          causal entries
//   capture_hits_kernel    one pass over the causal half of every map: per row the
//                          min/max, the exact float32 cut point x* of the decision
//                          t(x) >= tau, and the hit counts of every diagonal and column
//   capture_select_kernel  gamma = hits / cells in fp64, keep gamma >= mu, ordered
//                          compaction per map
//   capture_pack_kernel    CSR offsets across maps and the final lists
//
// Exactness.  The decision for an entry x is made by the sequence
//   z = x + eps; s = sqrt(z); y = (s - 1) / lambda; t = (y - y_lo) / (y_hi - y_lo); t >= tau
// in correctly rounded fp64 (lambda = 1 drops the sqrt; dividing by lambda = 1/2 is the
// exact scaling by 2), with y_lo / y_hi the same sequence at the row (or map) min / max.
// Every step is monotone non-decreasing in x, so for the non-negative floats of a row
// there is one cut point x* with decision(x) == (x >= x*).  The kernel finds x* exactly
// by evaluating the very same sequence on candidate floats: first the closed-form
// estimate and its neighbours (one lane per row), and only when the cut is not among
// them a window of 32 candidates and a 33-way bracketing search (the whole warp), so
// each decision equals the one obtained by evaluating the sequence at every entry.
// The division by y_hi - y_lo is filtered (see row_cut): only a quotient within a
// relative 2^-48 of tau takes the correctly rounded division.
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "trace.h"

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
    int64_t wait_ns;   // limit of each wait for a staged row
    int row_floats;    // floats of the rows a hits CTA keeps in shared memory (even)
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
    // lambda is 1/2 or 1 here: dividing by it is an exact scaling by 2 or 1
    if constexpr (TR == TR_SQRT) return __dmul_rn(__dsub_rn(__dsqrt_rn(z), 1.0), 2.0);
    if constexpr (TR == TR_LINEAR) return __dsub_rn(z, 1.0);
    if (lambda == 0.0) return log(z);
    return __ddiv_rn(__dsub_rn(pow(z, lambda), 1.0), lambda);
}

// The row's constants of the decision t = RN((y - y_lo) / y_range) >= tau.  The division
// is filtered: q = RN(a * RN(1 / y_range)) is within a relative 2^-52 of a / y_range when
// every quantity is a normal number, so q above tau (1 + 2^-48) proves a / y_range > tau
// (hence t >= tau) and q below tau (1 - 2^-48) proves a / y_range below the rounding
// boundary under tau (hence t < tau); only a q inside that band, or a row outside the
// normal range (use = false), takes the correctly rounded division.
struct RowCut {
    double ylo, yrange, rinv, thi, tlo, tau;
    bool use;
};

__device__ __forceinline__ RowCut row_cut(double ylo, double yhi, double tau) {
    RowCut c;
    c.ylo = ylo;
    c.yrange = __dsub_rn(yhi, ylo);
    c.tau = tau;
    const double at = fabs(tau);
    c.use = c.yrange >= 0x1p-1000 && c.yrange <= 0x1p1000 && at >= 0x1p-900 && at <= 0x1p900;
    c.rinv = c.use ? __drcp_rn(c.yrange) : 0.0;
    c.thi = tau + at * 0x1p-48;
    c.tlo = tau - at * 0x1p-48;
    return c;
}

template <int TR>
__device__ __forceinline__ bool decide(uint32_t xbits, double eps, double lambda, const RowCut &c) {
    const double x = static_cast<double>(__uint_as_float(xbits));
    const double a = __dsub_rn(box_cox_rn<TR>(x, eps, lambda), c.ylo);
    if (c.use) {
        const double q = __dmul_rn(a, c.rinv);
        if (q >= c.thi) return true;
        if (q < c.tlo) return false;
    }
    return __ddiv_rn(a, c.yrange) >= c.tau;
}

// Closed-form estimate of a row's cut point as a float bit pattern in [u0, u1] (the
// inverse of the transform at tau without rounding); it only chooses where the exact
// decision is evaluated first.
template <int TR>
__device__ __forceinline__ uint32_t cut_estimate(float mn, float mx, double eps, double lambda, double tau) {
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
    return __float_as_uint(ef);
}

// One lane's search for its own row's cut: the decision at the estimate and at its
// neighbours.  Returns true and sets *cut when the smallest float bit pattern u in
// [u0, u1] with decide(u) true (u1 + 1 if none) is among them; false otherwise (the
// warp-wide search then takes the row).
template <int TR>
__device__ __forceinline__ bool cut_near_estimate(uint32_t u0, uint32_t u1, float mn, float mx, double eps,
                                                  double lambda, double tau, uint32_t *cut) {
    const RowCut rc = row_cut(box_cox_rn<TR>(static_cast<double>(mn), eps, lambda),
                              box_cox_rn<TR>(static_cast<double>(mx), eps, lambda), tau);
    const uint32_t ue = cut_estimate<TR>(mn, mx, eps, lambda, tau);
    if (decide<TR>(ue, eps, lambda, rc)) {
        if (ue > u0 && decide<TR>(ue - 1, eps, lambda, rc)) return false;
        *cut = ue;
        return true;
    }
    if (ue < u1 && !decide<TR>(ue + 1, eps, lambda, rc)) return false;
    *cut = ue + 1;
    return true;
}

// Smallest float bit pattern u in [u0, u1] with decide(u) true, or u1 + 1 if none.
// Collective over the warp; every lane returns the same value.
template <int TR>
__device__ uint32_t find_cut(uint32_t u0, uint32_t u1, float mn, float mx, double eps, double lambda,
                             double tau) {
    const int lane = threadIdx.x & 31;
    const RowCut rc = row_cut(box_cox_rn<TR>(static_cast<double>(mn), eps, lambda),
                              box_cox_rn<TR>(static_cast<double>(mx), eps, lambda), tau);
    const int64_t ue = static_cast<int64_t>(cut_estimate<TR>(mn, mx, eps, lambda, tau));

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
        if (lane < np) val = decide<TR>(static_cast<uint32_t>(p), eps, lambda, rc);
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

// 1-D bulk copy (no multicast) of `bytes` from global memory into this CTA's shared
// memory, completing on `bar` with transaction bytes.  Both addresses 16-byte aligned,
// bytes a multiple of 16.
__device__ __forceinline__ void bulk_load_1d(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Bounded wait for a staged row: a non-blocking test first (a limit of 0 gives up when it
// fails), then sleeping in try_wait until the limit.
__device__ __forceinline__ bool row_wait(uint64_t *bar, uint32_t parity, int64_t limit_ns, volatile int *abort) {
    if (mbar_test(bar, parity)) return true;
    if (limit_ns <= 0) return false;
    return mbar_wait(bar, parity, limit_ns, abort);
}

// Bit t of the low byte of x moved to bit 4t.
__device__ __forceinline__ uint32_t spread4(uint32_t x) {
    x &= 0xffu;
    x = (x | (x << 12)) & 0x000f000fu;
    x = (x | (x << 6)) & 0x03030303u;
    x = (x | (x << 3)) & 0x11111111u;
    return x;
}

// Rows of a hits CTA: map m, rows i = chunk + row_chunks * r for r = 0 .. R - 1, each
// kept in shared memory at a 16-byte aligned offset (round4(i + 1) floats).  Warp w takes
// rows in snake order (w, 15 - w, 16 + w, 31 - w, ...), so that every warp's rows add
// up to about the same length.
__device__ __forceinline__ int snake_row(int t, int warp) {
    return kCaptureWarps * t + ((t & 1) ? kCaptureWarps - 1 - warp : warp);
}
constexpr int kHitsMaxRows = 128;
// Limit of each wait for a copy still in flight after a timeout (independent of the
// wait-limit knob, which may be 0): the CTA must not exit while a copy can still land
// in its shared memory.
constexpr int64_t kHitsDrainLimitNs = 1000000000LL;
__host__ __device__ __forceinline__ int round4(int x) { return (x + 3) & ~3; }

// Shared-memory bytes of a hits CTA whose rows hold `row_floats` floats in total.
__host__ __device__ inline size_t hits_smem_bytes(int L, int row_floats) {
    return sizeof(float) * static_cast<size_t>(row_floats) + 2 * sizeof(int32_t) * static_cast<size_t>(L) +
           kHitsMaxRows * (sizeof(uint64_t) + 4 * sizeof(uint32_t));
}

// One pass over the causal half of map m, rows interleaved over row_chunks CTAs.  The
// CTA first brings all of its rows into shared memory (BULK: one bulk copy per row of
// its first i + 1 entries rounded up to 16 bytes, still inside the row, each completing
// on its own mbarrier; otherwise plain loads), then works in three phases:
//   A  per row (one warp): the min and max bit patterns of the causal entries (for
//      non-negative floats the order of the bits is the order of the values; -0 is +0)
//   B  per row (one lane): the cut point x*, the smallest float with decision true,
//      by evaluating the exact decision at the closed-form estimate and its neighbours;
//      a row whose cut is elsewhere is searched by the whole warp (find_cut)
//   C  per row (one warp): the entries x >= x*; their diagonals counted with
//      shared-memory atomics, their columns in registers (a lane always holds the same
//      four columns of each 128-column block), and the true-mask words if requested.
// Lanes read four consecutive entries at a time (16-byte shared loads), 128 per warp.
// The per-row scalar work of phase B (transforms of the row's min and max, the estimate,
// three decisions) is spread over 32 rows per warp instruction.
template <int KB, int TR, bool BULK>
__global__ void __launch_bounds__(kCaptureThreads, 3)
    capture_hits_kernel(CaptureParams p) {
    extern __shared__ __align__(128) unsigned char s_raw[];
    const int L = p.L;
    float *s_rows = reinterpret_cast<float *>(s_raw);
    int32_t *s_diag = reinterpret_cast<int32_t *>(s_rows + p.row_floats);  // [L], then columns [L]
    int32_t *s_col = s_diag + L;
    uint64_t *s_bar = reinterpret_cast<uint64_t *>(s_diag + 2 * L);  // 8-byte aligned: L, row_floats even
    uint32_t *s_off = reinterpret_cast<uint32_t *>(s_bar + kHitsMaxRows);
    uint32_t *s_mn = s_off + kHitsMaxRows;
    uint32_t *s_mx = s_mn + kHitsMaxRows;
    uint32_t *s_cut = s_mx + kHitsMaxRows;
    __shared__ uint32_t s_map_cut;
    __shared__ int s_abort, s_bad;

    const int m = blockIdx.x / p.row_chunks;
    const int chunk = blockIdx.x % p.row_chunks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = chunk < L ? (L - 1 - chunk) / p.row_chunks + 1 : 0;
    const float *map = p.maps + static_cast<size_t>(m) * L * L;
    if (warp == 0) {
        // row offsets (a warp prefix sum), barriers, then one bulk copy per row
        uint32_t base = 0;
        for (int r0 = 0; r0 < R; r0 += 32) {
            const int r = r0 + lane;
            const uint32_t sz = r < R ? static_cast<uint32_t>(round4(chunk + p.row_chunks * r + 1)) : 0u;
            uint32_t x = sz;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (r < R) {
                s_off[r] = base + x - sz;
                if (BULK) mbar_init(&s_bar[r], 1);
            }
            base += __shfl_sync(0xffffffffu, x, 31);
        }
        if (BULK) {
            fence_barrier_init();
            __syncwarp();
            for (int r = lane; r < R; r += 32) {
                const int i = chunk + p.row_chunks * r;
                const uint32_t bytes = 4u * static_cast<uint32_t>(round4(i + 1));
                mbar_arrive_expect_tx(&s_bar[r], bytes);
                bulk_load_1d(s_rows + s_off[r], map + static_cast<size_t>(i) * L, bytes, &s_bar[r]);
            }
        }
    }
    for (int k = threadIdx.x; k < 2 * L; k += kCaptureThreads) s_diag[k] = 0;
    if (threadIdx.x == 0) {
        s_abort = 0;
        s_bad = 0;
    }
    __syncthreads();
    if (!BULK) {
        for (int r = warp; r < R; r += kCaptureWarps) {
            const int i = chunk + p.row_chunks * r;
            const float *row = map + static_cast<size_t>(i) * L;
            float *dst = s_rows + s_off[r];
#pragma unroll 4
            for (int j = lane; j <= i; j += 32) dst[j] = __ldg(row + j);
        }
        __syncthreads();
    }
    // per-map scaling: one cut for the whole map, from its min and max (warp 0)
    if (p.scaling == 1 && warp == 0) {
        const float mn = __uint_as_float(p.map_mm[2 * m]), mx = __uint_as_float(p.map_mm[2 * m + 1]);
        const uint32_t u0 = __float_as_uint(mn), u1 = __float_as_uint(mx);
        const uint32_t c = (u0 == u1) ? ((1.0 >= p.tau) ? 0u : 0xffffffffu)
                                      : find_cut<TR>(u0, u1, mn, mx, p.eps, p.lambda, p.tau);
        if (lane == 0) s_map_cut = c;
    }

    // ---- A: min / max bit patterns of each row's causal entries ----
    bool bad = false;
    for (int t = 0;; ++t) {
        const int r = snake_row(t, warp);
        if (r >= R) break;
        const int i = chunk + p.row_chunks * r, n = i + 1;
        if (BULK) {
            const bool ok = row_wait(&s_bar[r], 0, p.wait_ns, &s_abort);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) {
                    s_abort = 1;
                    report(p.status, SSA_ERR_TIMEOUT);
                }
                break;
            }
        }
        const float *buf = s_rows + s_off[r];
        uint32_t mn = 0xffffffffu, amx = 0u, rmx = 0u;
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            const int j0 = 128 * k + 4 * lane;
            // warp-uniform: whole blocks below the diagonal, the block that holds it, and
            // blocks past it (skipped)
            if (128 * (k + 1) <= n) {
                const uint4 v = *reinterpret_cast<const uint4 *>(buf + j0);
                const uint32_t b[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t a = b[q] & 0x7fffffffu;  // -0 counts as +0
                    mn = min(mn, a);
                    amx = max(amx, a);
                    rmx = max(rmx, b[q]);
                }
            } else if (128 * k < n && j0 < n) {
                const uint4 v = *reinterpret_cast<const uint4 *>(buf + j0);
                const uint32_t b[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (j0 + q < n) {
                        const uint32_t a = b[q] & 0x7fffffffu;
                        mn = min(mn, a);
                        amx = max(amx, a);
                        rmx = max(rmx, b[q]);
                    }
                }
            }
        }
        // negative (other than -0), infinite or NaN entries
        bad |= amx > 0x7f7fffffu || rmx > 0x80000000u;
        mn = __reduce_min_sync(0xffffffffu, mn);
        amx = __reduce_max_sync(0xffffffffu, amx);
        if (lane == 0) {
            s_mn[r] = mn;
            s_mx[r] = amx;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) s_bad = 1;
    __syncthreads();

    // ---- B: each row's cut point, one lane per row ----
    if (!s_abort && p.scaling != 1) {
        for (int r0 = 32 * warp; r0 < R; r0 += 32 * kCaptureWarps) {
            const int r = r0 + lane;
            uint32_t cut = 0u;
            bool done = true;
            uint32_t u0 = 0u, u1 = 0u;
            if (r < R) {
                u0 = s_mn[r];
                u1 = s_mx[r];
                if (u0 == u1) cut = (1.0 >= p.tau) ? 0u : 0xffffffffu;  // constant row: t = 1
                else
                    done = cut_near_estimate<TR>(u0, u1, __uint_as_float(u0), __uint_as_float(u1), p.eps,
                                                 p.lambda, p.tau, &cut);
            }
            // rows whose cut is not next to the estimate: searched by the whole warp
            uint32_t pending = __ballot_sync(0xffffffffu, !done);
            while (pending) {
                const int src = __ffs(pending) - 1;
                pending &= pending - 1;
                const uint32_t a0 = __shfl_sync(0xffffffffu, u0, src), a1 = __shfl_sync(0xffffffffu, u1, src);
                const uint32_t c = find_cut<TR>(a0, a1, __uint_as_float(a0), __uint_as_float(a1), p.eps, p.lambda,
                                                p.tau);
                if (lane == src) cut = c;
            }
            if (r < R) s_cut[r] = cut;
        }
    }
    __syncthreads();

    // ---- C: hits per diagonal (shared atomics) and column (registers), true-mask words ----
    uint32_t cnt[KB];  // four 8-bit column counters per block (at most 128 rows per CTA)
#pragma unroll
    for (int k = 0; k < KB; ++k) cnt[k] = 0u;
    if (!s_abort) {
        for (int t = 0;; ++t) {
            const int r = snake_row(t, warp);
            if (r >= R) break;
            const int i = chunk + p.row_chunks * r, n = i + 1;
            // x >= x* compared as floats: for the non-negative floats of a row the same as
            // comparing bit patterns, with -0 equal to +0, and a cut of 0xffffffff (NaN)
            // keeps none
            const float xcut = __uint_as_float(p.scaling == 1 ? s_map_cut : s_cut[r]);
            const float *buf = s_rows + s_off[r];
            uint32_t *bits_row = p.bits ? p.bits + (static_cast<size_t>(m) * L + i) * p.bits_words : nullptr;
#pragma unroll
            for (int k = 0; k < KB; ++k) {
                const int j0 = 128 * k + 4 * lane;
                bool on[4] = {false, false, false, false};
                if (128 * k < n && j0 < n) {
                    const float4 v = *reinterpret_cast<const float4 *>(buf + j0);
                    const float x[4] = {v.x, v.y, v.z, v.w};
                    if (128 * (k + 1) <= n) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) on[q] = x[q] >= xcut;
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) on[q] = j0 + q < n && x[q] >= xcut;
                    }
                    int32_t *dg = s_diag + (i - j0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (on[q]) {
                            cnt[k] += 1u << (8 * q);
                            atomicAdd(dg - q, 1);
                        }
                    }
                }
                if (bits_row && 4 * k < p.bits_words) {
                    // word 4k + w holds columns 128k + 32w .. + 31: lanes 8w .. 8w + 7
                    uint32_t ball[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) ball[q] = __ballot_sync(0xffffffffu, on[q]);
                    if (lane < 4 && 4 * k + lane < p.bits_words) {
                        uint32_t word = 0u;
#pragma unroll
                        for (int q = 0; q < 4; ++q) word |= spread4(ball[q] >> (8 * lane)) << q;
                        bits_row[4 * k + lane] = word;
                    }
                }
            }
        }
    }
    // the lanes' column counts into the shared column histogram
#pragma unroll
    for (int k = 0; k < KB; ++k) {
        if (cnt[k]) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t c = (cnt[k] >> (8 * q)) & 0xffu;
                if (c) atomicAdd(&s_col[128 * k + 4 * lane + q], static_cast<int32_t>(c));
            }
        }
    }
    __syncthreads();
    if (BULK && s_abort && threadIdx.x == 0) {
        // a row copy did not land within the wait limit: wait (again bounded) for every
        // copy of this CTA before it may exit
        for (int r = 0; r < R; ++r)
            if (!mbar_wait(&s_bar[r], 0, kHitsDrainLimitNs, nullptr)) break;
    }
    if (threadIdx.x == 0 && s_bad) report(p.status, SSA_ERR_INVALID);
    if (s_abort) return;
    int32_t *hits = p.hits + static_cast<size_t>(m) * 2 * L;
    for (int k = threadIdx.x; k < 2 * L; k += kCaptureThreads) {
        const int v = s_diag[k];
        if (v) atomicAdd(hits + k, v);
    }
}

// Launch of one instantiation of the hits kernel; the shared-memory opt-in above 48 KB is
// made once per device, for the largest CTA the host ever plans (kHitsSmemMax).
constexpr size_t kHitsSmemMax = 75 * 1024;

template <int KB, int TR, bool BULK>
int launch_hits_kernel(const CaptureParams &p, unsigned grid, size_t smem, cudaStream_t s) {
    static std::atomic<uint64_t> ready{0};
    if (smem > 48 * 1024) {
        int dev = 0;
        SSA_CUDA_TRY(cudaGetDevice(&dev));
        const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0;
        if (!bit || !(ready.load() & bit)) {
            SSA_CUDA_TRY(cudaFuncSetAttribute(capture_hits_kernel<KB, TR, BULK>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(kHitsSmemMax)));
            ready.fetch_or(bit);
        }
    }
    capture_hits_kernel<KB, TR, BULK><<<grid, kCaptureThreads, smem, s>>>(p);
    SSA_LAUNCH_CHECK();
    return SSA_OK;
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
template <bool VEC>
__global__ void __launch_bounds__(kCaptureThreads) capture_minmax_kernel(CaptureParams p) {
    const int L = p.L;
    const int m = blockIdx.x / p.row_chunks;
    const int chunk = blockIdx.x % p.row_chunks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *map = p.maps + static_cast<size_t>(m) * L * L;
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (int i = chunk + p.row_chunks * warp; i < L; i += p.row_chunks * kCaptureWarps) {
        const float *row = map + static_cast<size_t>(i) * L;
        if (VEC) {
            // 16-byte loads of four entries (rows start on 16-byte boundaries), unrolled
            // so that several are in flight at once
#pragma unroll 4
            for (int j0 = 4 * lane; j0 <= i; j0 += 128) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(row + j0));
                const uint32_t b[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (j0 + q <= i) {
                        const uint32_t a = b[q] & 0x7fffffffu;  // -0 counts as +0
                        mn = min(mn, a);
                        mx = max(mx, a);
                    }
                }
            }
        } else {
#pragma unroll 8
            for (int j = lane; j <= i; j += 32) {
                const uint32_t a = __float_as_uint(__ldg(row + j)) & 0x7fffffffu;
                mn = min(mn, a);
                mx = max(mx, a);
            }
        }
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
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
    ssa::TraceRange trace_range("sparse_pattern_capture_ex");
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
    // Rows are staged by bulk copies when every row starts on a 16-byte boundary.
    const bool bulk = (L % 4 == 0) && ((reinterpret_cast<uintptr_t>(maps) & 15u) == 0);
    p.wait_ns = wait_limit_ns();
    // Enough CTAs to fill the GPU a few times over even for a few maps (each warp then
    // takes fewer rows); then as many as it takes for each CTA's rows to fit its shared
    // memory (three CTAs per SM).
    int chunks = 8;
    while (chunks < 64 && static_cast<long long>(n_maps) * chunks < 4LL * sm_count_capture() &&
           chunks * 2 * kCaptureWarps <= L)
        chunks *= 2;
    auto row_floats = [L](int c) {  // the most any CTA keeps, rounded up to an even count
        int most = 0;
        for (int ch = 0; ch < c && ch < L; ++ch) {
            int f = 0;
            for (int i = ch; i < L; i += c) f += round4(i + 1);
            most = f > most ? f : most;
        }
        return most + (most & 1);
    };
    int rf = row_floats(chunks);
    while ((L + chunks - 1) / chunks > kHitsMaxRows || hits_smem_bytes(L, rf) > kHitsSmemMax) {
        chunks *= 2;
        rf = row_floats(chunks);
    }
    p.row_chunks = chunks;
    p.row_floats = rf;
    const size_t smem = hits_smem_bytes(L, rf);
    const unsigned grid = static_cast<unsigned>(n_maps) * chunks;
    if (scaling == SSA_SCALE_MAP) {
        capture_minmax_init_kernel<<<(n_maps + 255) / 256, 256, 0, s>>>(p.map_mm, n_maps);
        SSA_LAUNCH_CHECK();
        if (bulk) capture_minmax_kernel<true><<<grid, kCaptureThreads, 0, s>>>(p);
        else capture_minmax_kernel<false><<<grid, kCaptureThreads, 0, s>>>(p);
        SSA_LAUNCH_CHECK();
    }
    const int tr = lambda == 0.5 ? TR_SQRT : (lambda == 1.0 ? TR_LINEAR : TR_POW);
    // KB: 128-column blocks of a row
    auto launch_hits = [&](auto KBC, auto BK) -> int {
        constexpr int KB = decltype(KBC)::value;
        constexpr bool BULK = decltype(BK)::value;
        if (tr == TR_SQRT) return launch_hits_kernel<KB, TR_SQRT, BULK>(p, grid, smem, s);
        if (tr == TR_LINEAR) return launch_hits_kernel<KB, TR_LINEAR, BULK>(p, grid, smem, s);
        return launch_hits_kernel<KB, TR_POW, BULK>(p, grid, smem, s);
    };
    using K4 = std::integral_constant<int, 4>;
    using K8 = std::integral_constant<int, 8>;
    using Bulk = std::true_type;
    using Plain = std::false_type;
    const int rc = L <= 512 ? (bulk ? launch_hits(K4{}, Bulk{}) : launch_hits(K4{}, Plain{}))
                            : (bulk ? launch_hits(K8{}, Bulk{}) : launch_hits(K8{}, Plain{}));
    if (rc != SSA_OK) return rc;
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
    ssa::TraceRange trace_range("sparse_pattern_capture_noalloc");
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
