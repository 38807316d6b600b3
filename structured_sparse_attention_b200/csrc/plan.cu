// plan.cu -- stage two of DAM: extension of the kept patterns to S x S and their
// compilation into per-query-block key-tile lists (DAM review page, "What carries
// the argument": the kept patterns are pasted into an S x S mask; "Circularity
// Check" step 1: the mask is the union of the matched patterns).
//
// In list form the extension keeps every diagonal r < S and every column c < S.  The
// tile plan is this library's own layout of that mask for the attention kernel:
// for each (head, query block) the ascending 128-key windows the band reaches (each
// starting where the band's keys start, not at a multiple of 128), each with a
// 255-bit local-diagonal mask, a 128-bit column-exclusion mask and a FULL flag, plus
// the number of columns the stripe phase covers (exact semantics in ssa.h).
//
// Kernels (one warp per (head, query block) for the tile work)
//   validate_lists_kernel  lists sorted, unique, non-negative; kept counts r < S, c < S
//   exclusive_scan_kernel  single-block scan (list offsets, tile offsets; exact 64-bit
//                          total)
//   extend_copy_kernel     the extended CSR lists
//   run_start_kernel       per head: first index of the run (offsets <= 128 apart)
//                          holding each kept diagonal
//   plan_tiles_kernel      count pass / fill pass of the band windows + stripe counts
//   plan_totals_kernel     totals for the sizing pass
//   plan_check_kernel      fill pass: the lists and the tiles fit the plan's capacities,
//                          else the kernels that write the plan return at once (the plan
//                          keeps its previous content) and SSA_ERR_CAPACITY is reported
//
// Fill pass order: everything that sizes the new plan (validation, list scans, run
// starts, tile counts, tile scan) writes only the workspace; the capacity check follows;
// only then are the plan's lists and tiles written (tile_ptr by the fill kernel).
#include "common.cuh"
#include "trace.h"

namespace ssa {
namespace {

constexpr int kTile = SSA_BLOCK;
constexpr int kScanThreads = 1024;

struct Totals {  // device-side result of the sizing pass
    int32_t status;
    int32_t n_diag;
    int32_t n_vert;
    int32_t max_vert;
    int64_t n_tiles;  // exact total of the tile scan
    int32_t abort;    // fill pass: the new plan does not fit; nothing of the plan is written
};

struct PlanParams {
    int H, S, nqb;
    const int32_t *dptr, *doff, *vptr, *vcol;  // input lists
    int32_t *ext_counts;   // [2H]: kept diagonals, kept columns per head
    int32_t *ext_scan;     // [2 (H+1)]: exclusive scans of the two count arrays
    int32_t *tile_counts;  // [H*nqb]
    int32_t *run0;         // [H][S]: run start index of each kept diagonal
    int32_t *tile_pos;     // [H*nqb + 1] workspace: exclusive scan of tile_counts
    int32_t *tile_ptr;     // [H*nqb + 1] fill pass: the plan's copy of tile_pos
    Totals *totals;
    int32_t *ws_status;
    int32_t *dev_status;
    // fill pass outputs
    int64_t capacity;
    int32_t cap_diag, cap_vert, cap_max_vert;  // list capacities of the plan
    int32_t *tile_key0;
    uint64_t *tile_dmask;
    uint64_t *tile_cmask;
    uint32_t *tile_flags;
    int32_t *stripe_cnt;
    int32_t *ext_dptr, *ext_doff, *ext_vptr, *ext_vcol;
    // Case 2 (tmask non-null): the true masks [H][L][bw] and the bitmap tiles
    const uint32_t *tmask;
    int L, bw;      // capture length, words per true-mask row (ceil(L / 32))
    int nL, slots;  // query blocks holding a row < min(L, S); bitmap slots per head
    uint64_t *tile_bits;
};

__global__ void validate_lists_kernel(PlanParams p) {
    const int h = blockIdx.x;
    const int32_t *D = p.doff + p.dptr[h];
    const int32_t *C = p.vcol + p.vptr[h];
    const int nd = p.dptr[h + 1] - p.dptr[h];
    const int nc = p.vptr[h + 1] - p.vptr[h];
    bool bad = nd < 0 || nc < 0;
    for (int k = threadIdx.x; !bad && k < nd; k += blockDim.x)
        if (D[k] < 0 || (k > 0 && D[k] <= D[k - 1])) bad = true;
    for (int k = threadIdx.x; !bad && k < nc; k += blockDim.x)
        if (C[k] < 0 || (k > 0 && C[k] <= C[k - 1])) bad = true;
    if (__syncthreads_or(bad)) {
        if (threadIdx.x == 0) {
            report(p.ws_status, SSA_ERR_INVALID);
            report(p.dev_status, SSA_ERR_INVALID);
            p.ext_counts[2 * h] = 0;
            p.ext_counts[2 * h + 1] = 0;
        }
        return;
    }
    if (threadIdx.x == 0) {
        p.ext_counts[2 * h] = lower_bound_i32(D, nd, p.S);
        p.ext_counts[2 * h + 1] = lower_bound_i32(C, nc, p.S);
    }
}

// out[k] = sum_{k' < k} in[k' * stride + offset] for k in [0, n] (inputs >= 0); one
// block.  Sums are taken in 64 bits: out[] holds them clamped to INT32_MAX, and *total
// (may be null) the exact sum of all n, so that a caller can tell an int32 overflow
// from a fit.  Chunks of kScanThreads x kScanPer elements: each thread loads kScanPer
// consecutive elements at once (all loads in flight together), then one block scan of
// the threads' sums.
constexpr int kScanPer = 8;
__device__ __forceinline__ int32_t clamp_i32(int64_t x) {
    return static_cast<int32_t>(x < INT32_MAX ? x : INT32_MAX);
}
__global__ void __launch_bounds__(kScanThreads)
    exclusive_scan_kernel(const int32_t *in, int n, int stride, int offset, int32_t *out, int64_t *total) {
    __shared__ int64_t s_warp[kScanThreads / 32];
    __shared__ int64_t s_carry;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int start = 0; start < n; start += kScanThreads * kScanPer) {
        const int k0 = start + threadIdx.x * kScanPer;
        int v[kScanPer];
#pragma unroll
        for (int t = 0; t < kScanPer; ++t) {
            const int k = k0 + t;
            v[t] = k < n ? in[static_cast<size_t>(k) * stride + offset] : 0;
        }
        int64_t sum = 0;
#pragma unroll
        for (int t = 0; t < kScanPer; ++t) sum += v[t];
        int64_t x = sum;  // inclusive scan of the threads' sums within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {  // exclusive scan of the warp totals
            const int64_t w = lane < kScanThreads / 32 ? s_warp[lane] : 0;
            int64_t y = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int64_t z = __shfl_up_sync(0xffffffffu, y, o);
                if (lane >= o) y += z;
            }
            if (lane < kScanThreads / 32) s_warp[lane] = y - w;
        }
        __syncthreads();
        int64_t run = s_carry + s_warp[warp] + x - sum;  // before this thread's first element
#pragma unroll
        for (int t = 0; t < kScanPer; ++t) {
            const int k = k0 + t;
            if (k < n) out[k] = clamp_i32(run);
            run += v[t];
        }
        __syncthreads();
        if (threadIdx.x == kScanThreads - 1) s_carry = run;  // the last thread's end: the chunk total
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        out[n] = clamp_i32(s_carry);
        if (total) *total = s_carry;
    }
}

__global__ void extend_copy_kernel(PlanParams p) {
    if (p.totals->abort) return;
    const int h = blockIdx.x;
    const int32_t *D = p.doff + p.dptr[h];
    const int32_t *C = p.vcol + p.vptr[h];
    const int nd = p.ext_counts[2 * h], nc = p.ext_counts[2 * h + 1];
    const int od = p.ext_scan[h], oc = p.ext_scan[(p.H + 1) + h];
    for (int k = threadIdx.x; k < nd; k += blockDim.x) p.ext_doff[od + k] = D[k];
    for (int k = threadIdx.x; k < nc; k += blockDim.x) p.ext_vcol[oc + k] = C[k];
    if (threadIdx.x == 0) {
        p.ext_dptr[h] = od;
        p.ext_vptr[h] = oc;
        if (h == p.H - 1) {
            p.ext_dptr[h + 1] = od + nd;
            p.ext_vptr[h + 1] = oc + nc;
        }
    }
}

// run0[k] = the largest k' <= k with k' == 0 or D[k'] - D[k'-1] > 128: the first index of
// the run of offsets (each within 128 of the previous one) that holds D[k].  A run
// reaches one contiguous range of keys from the 128 rows of a query block.  One block
// per head: an inclusive max-scan of the run boundaries.
__global__ void __launch_bounds__(kScanThreads) run_start_kernel(PlanParams p) {
    __shared__ int32_t s_warp[kScanThreads / 32];
    __shared__ int32_t s_carry;
    const int h = blockIdx.x;
    const int32_t *D = p.doff + p.dptr[h];
    const int nd = p.ext_counts[2 * h];
    int32_t *run0 = p.run0 + static_cast<size_t>(h) * p.S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int start = 0; start < nd; start += kScanThreads) {
        const int k = start + threadIdx.x;
        int x = (k < nd && (k == 0 || __ldg(D + k) - __ldg(D + k - 1) > kTile)) ? k : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) x = max(x, __shfl_up_sync(0xffffffffu, x, o) * (lane >= o ? 1 : 0));
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        int before = s_carry, total = s_carry;
        for (int w = 0; w < kScanThreads / 32; ++w) {
            if (w < warp) before = max(before, s_warp[w]);
            total = max(total, s_warp[w]);
        }
        if (k < nd) run0[k] = max(x, before);
        __syncthreads();
        if (threadIdx.x == 0) s_carry = total;
        __syncthreads();
    }
}

__device__ __forceinline__ void set_bit_range(uint64_t (&w)[4], int a, int b) {  // inclusive
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int lo = max(a, 64 * k), hi = min(b, 64 * k + 63);
        if (lo <= hi) {
            const int n = hi - lo + 1;
            const uint64_t bits = (n == 64) ? ~0ull : (((1ull << n) - 1ull) << (lo - 64 * k));
            w[k] |= bits;
        }
    }
}

// Evaluate the window of keys key0 .. key0+127 for query block qb of one head.
// Returns 0 (not listed), 1 (listed), 2 (FULL).
__device__ int eval_window(const int32_t *D, int nD, const int32_t *C, int nC, int S, int qb, int key0,
                           uint64_t (&dm)[4], uint64_t (&cm)[2]) {
    const int base = kTile * qb - key0 - (kTile - 1);  // r of dmask bit 0
    const int lb = lower_bound_i32(D, nD, max(base, 0));
    const int ub = lower_bound_i32(D, nD, base + 2 * kTile - 1);
    if (lb == ub) return 0;
    dm[0] = dm[1] = dm[2] = dm[3] = 0;
    const int dfirst = __ldg(D + lb), dlast = __ldg(D + ub - 1);
    if (dlast - dfirst == ub - 1 - lb) {
        set_bit_range(dm, dfirst - base, dlast - base);  // a contiguous run of offsets
    } else {
        for (int k = lb; k < ub; ++k) {
            const int t = __ldg(D + k) - base;
            dm[t >> 6] |= 1ull << (t & 63);
        }
    }
    cm[0] = cm[1] = 0;
    const int cl = lower_bound_i32(C, nC, key0);
    for (int k = cl; k < nC; ++k) {
        const int jl = __ldg(C + k) - key0;
        if (jl >= kTile) break;
        cm[jl >> 6] |= 1ull << (jl & 63);
    }
    const int nrows = min(kTile, S - kTile * qb);
    bool listed = false;
    if ((cm[0] | cm[1]) == 0) {
        // with no excluded column, diagonal t has a cell in a valid row iff t <= nrows + 126
        uint64_t lim[4] = {0, 0, 0, 0};
        set_bit_range(lim, 0, nrows + kTile - 2);
        listed = ((dm[0] & lim[0]) | (dm[1] & lim[1]) | (dm[2] & lim[2]) | (dm[3] & lim[3])) != 0;
    } else {
        for (int il = 0; il < nrows && !listed; ++il) {
            uint64_t lo, hi;
            row_diag_mask(dm, il, lo, hi);
            listed = ((lo & ~cm[0]) | (hi & ~cm[1])) != 0;
        }
    }
    if (!listed) return 0;
    const bool all = dm[0] == ~0ull && dm[1] == ~0ull && dm[2] == ~0ull && dm[3] == (~0ull >> 1);
    // all 255 offsets present implies r >= 0 everywhere, i.e. the window is left of the diagonal
    const bool full = kTile * (qb + 1) <= S && all && (cm[0] | cm[1]) == 0;
    return full ? 2 : 1;
}

// Diagonal and column masks of the window key0 .. key0 + 127 for query block qb (the
// dmask / cmask of eval_window, without its listing decision).
__device__ void window_masks(const int32_t *D, int nD, const int32_t *C, int nC, int qb, int key0,
                             uint64_t (&dm)[4], uint64_t (&cm)[2]) {
    const int base = kTile * qb - key0 - (kTile - 1);  // r of dmask bit 0
    const int lb = lower_bound_i32(D, nD, max(base, 0));
    const int ub = lower_bound_i32(D, nD, base + 2 * kTile - 1);
    dm[0] = dm[1] = dm[2] = dm[3] = 0;
    for (int k = lb; k < ub; ++k) {
        const int t = __ldg(D + k) - base;
        dm[t >> 6] |= 1ull << (t & 63);
    }
    cm[0] = cm[1] = 0;
    for (int k = lower_bound_i32(C, nC, key0); k < nC; ++k) {
        const int jl = __ldg(C + k) - key0;
        if (jl >= kTile) break;
        cm[jl >> 6] |= 1ull << (jl & 63);
    }
}

// Case 2, one warp per query block qb < nL of head h: element-bitmap tiles for the key
// blocks kb = 0..qb (key0 = 128 kb), listed when any cell is set.  Cell (i, j) of a tile:
// i < S and j <= i and, for i < L, bit j of row i of the head's true mask; for i >= L,
// i - j an extended diagonal or j an extended column.  Returns the tiles listed.
template <bool FILL>
__device__ int bitmap_tiles(const PlanParams &p, int h, int qb, const int32_t *D, int nD, const int32_t *C,
                            int nC, int64_t pos) {
    const int lane = threadIdx.x & 31;
    const int lo = kTile * qb;
    const uint32_t *tm = p.tmask + static_cast<size_t>(h) * p.L * p.bw;
    int count = 0;
    for (int kb = 0; kb <= qb; ++kb) {
        uint64_t dm[4], cm[2];
        const bool past_L = lo + kTile > p.L;  // the block holds rows >= L
        if (past_L) window_masks(D, nD, C, nC, qb, kTile * kb, dm, cm);
        uint64_t rb[4][2];
        uint64_t any = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int il = lane + 32 * q, i = lo + il;
            uint64_t b0 = 0, b1 = 0;
            if (i < p.S) {
                if (i < p.L) {
                    uint32_t w[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const int wi = 4 * kb + x;  // word of columns 32 wi .. 32 wi + 31
                        w[x] = wi < p.bw ? __ldg(tm + static_cast<size_t>(i) * p.bw + wi) : 0u;
                    }
                    b0 = static_cast<uint64_t>(w[0]) | (static_cast<uint64_t>(w[1]) << 32);
                    b1 = static_cast<uint64_t>(w[2]) | (static_cast<uint64_t>(w[3]) << 32);
                } else {
                    row_diag_mask(dm, il, b0, b1);  // diagonals (r >= 0, so j <= i)
                    b0 |= cm[0];
                    b1 |= cm[1];
                }
                if (kb == qb) {  // the diagonal tile: columns jl <= il only
                    const int n = il + 1;
                    b0 &= n >= 64 ? ~0ull : ((1ull << n) - 1ull);
                    b1 &= n >= 128 ? ~0ull : (n <= 64 ? 0ull : ((1ull << (n - 64)) - 1ull));
                }
            }
            rb[q][0] = b0;
            rb[q][1] = b1;
            any |= b0 | b1;
        }
        const int slot = h * p.slots + qb * (qb + 1) / 2 + kb;
        if (FILL) {  // every slot is written, listed or not
            uint64_t *bits = p.tile_bits + static_cast<size_t>(slot) * kTile * 2;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int il = lane + 32 * q;
                bits[2 * il] = rb[q][0];
                bits[2 * il + 1] = rb[q][1];
            }
        }
        if (!__any_sync(0xffffffffu, any != 0)) continue;
        if (FILL) {
            const int64_t t = pos + count;
            if (t < p.capacity) {
                if (lane == 0) {
                    p.tile_key0[t] = kTile * kb;
                    uint64_t *dst = p.tile_dmask + 4 * t;
                    dst[0] = static_cast<uint64_t>(slot);  // the bitmap's slot
                    dst[1] = dst[2] = dst[3] = 0;
                    p.tile_cmask[2 * t] = p.tile_cmask[2 * t + 1] = 0;
                    p.tile_flags[t] = 2u;  // BITMAP
                }
            } else if (lane == 0) {
                report(p.dev_status, SSA_ERR_CAPACITY);
            }
        }
        ++count;
    }
    return count;
}

// One warp per (head, query block).  FILL = false: count; FILL = true: write the tiles
// at the offsets of the tile scan and copy those offsets into the plan's tile_ptr.
template <bool FILL>
__global__ void __launch_bounds__(128) plan_tiles_kernel(PlanParams p) {
    const int item = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int items = p.H * p.nqb;
    if (item >= items || (FILL && p.totals->abort)) return;
    if (FILL && lane == 0) {
        p.tile_ptr[item] = p.tile_pos[item];
        if (item == items - 1) p.tile_ptr[items] = p.tile_pos[items];
    }
    const int h = item / p.nqb, qb = item % p.nqb;
    const int32_t *D = p.doff + p.dptr[h];
    const int32_t *C = p.vcol + p.vptr[h];
    const int nD = p.ext_counts[2 * h], nC = p.ext_counts[2 * h + 1];
    if (p.tmask && qb < p.nL) {  // Case 2: element-bitmap tiles, no stripe tiles
        const int n = bitmap_tiles<FILL>(p, h, qb, D, nD, C, nC, FILL ? p.tile_pos[item] : 0);
        if (lane == 0) {
            if (FILL) p.stripe_cnt[item] = 0;
            else p.tile_counts[item] = n;
        }
        return;
    }
    // windows are chosen over all 128 rows of the block (lo .. hi), even past S
    const int lo = kTile * qb, hi = lo + kTile - 1;
    if (FILL && lane == 0) p.stripe_cnt[item] = lower_bound_i32(C, nC, min(hi, p.S - 1) + 1);
    const int32_t *run0 = p.run0 + static_cast<size_t>(h) * p.S;
    // Runs of offsets from the largest r <= hi down, i.e. in ascending keys: run [ra, rb]
    // reaches keys [max(0, lo - rb), hi - ra]; windows step 128 keys from the larger of
    // that start and the end of the previous window.
    int k = lower_bound_i32(D, nD, hi + 1) - 1;
    int next = 0;
    int count = 0;
    int64_t pos = FILL ? p.tile_pos[item] : 0;
    while (k >= 0) {
        const int ks = run0[k];
        const int a = max(0, lo - __ldg(D + k)), b = hi - __ldg(D + ks);
        const int s0 = max(a, next);
        if (s0 <= b) {
            const int nw = (b - s0) / kTile + 1;
            for (int w0 = 0; w0 < nw; w0 += 32) {
                const int w = w0 + lane;
                const int key0 = s0 + kTile * w;
                uint64_t dm[4], cm[2];
                int r = 0;
                if (w < nw) r = eval_window(D, nD, C, nC, p.S, qb, key0, dm, cm);
                const uint32_t ball = __ballot_sync(0xffffffffu, r != 0);
                if (FILL && r) {
                    const int64_t t = pos + __popc(ball & ((1u << lane) - 1u));
                    if (t < p.capacity) {
                        p.tile_key0[t] = key0;
                        uint64_t *dst = p.tile_dmask + 4 * t;
                        dst[0] = dm[0];
                        dst[1] = dm[1];
                        dst[2] = dm[2];
                        dst[3] = dm[3];
                        p.tile_cmask[2 * t] = cm[0];
                        p.tile_cmask[2 * t + 1] = cm[1];
                        p.tile_flags[t] = (r == 2) ? 1u : 0u;
                    } else {
                        report(p.dev_status, SSA_ERR_CAPACITY);
                    }
                }
                pos += __popc(ball);
                count += __popc(ball);
            }
            next = s0 + kTile * nw;
        }
        k = ks - 1;
    }
    if (!FILL && lane == 0) p.tile_counts[item] = count;
}

// Fill pass: the new plan must fit the plan's arrays (sized by an earlier sizing pass):
// total diagonals, total columns, each head's columns within max_vert (the attention
// workspace's stripe buffers) and the tiles within n_tiles (and int32 offsets).
// Otherwise the kernels that write the plan return at once.
__global__ void __launch_bounds__(256) plan_check_kernel(PlanParams p) {
    __shared__ int s_bad;
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    bool bad = false;
    for (int h = threadIdx.x; h < p.H; h += blockDim.x) bad |= p.ext_counts[2 * h + 1] > p.cap_max_vert;
    if (bad) s_bad = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
        const int nd = p.ext_scan[p.H], nc = p.ext_scan[(p.H + 1) + p.H];
        const int64_t nt = p.totals->n_tiles;
        if (s_bad || nd > p.cap_diag || nc > p.cap_vert || nt > p.capacity || nt > INT32_MAX) {
            p.totals->abort = 1;
            report(p.dev_status, SSA_ERR_CAPACITY);
        }
    }
}

// Sizing pass: list totals and the largest column count (n_tiles comes from the tile scan).
__global__ void plan_totals_kernel(PlanParams p) {
    __shared__ int32_t s[3][32];
    int nd = 0, nv = 0, mv = 0;
    for (int h = threadIdx.x; h < p.H; h += blockDim.x) {
        nd += p.ext_counts[2 * h];
        nv += p.ext_counts[2 * h + 1];
        mv = max(mv, p.ext_counts[2 * h + 1]);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        nd += __shfl_xor_sync(0xffffffffu, nd, o);
        nv += __shfl_xor_sync(0xffffffffu, nv, o);
        mv = max(mv, __shfl_xor_sync(0xffffffffu, mv, o));
    }
    if (lane == 0) {
        s[0][warp] = nd;
        s[1][warp] = nv;
        s[2][warp] = mv;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        nd = nv = mv = 0;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
            nd += s[0][w];
            nv += s[1][w];
            mv = max(mv, s[2][w]);
        }
        p.totals->status = *p.ws_status;
        p.totals->n_diag = nd;
        p.totals->n_vert = nv;
        p.totals->max_vert = mv;
    }
}

size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace
}  // namespace ssa

using namespace ssa;

extern "C" size_t sparse_pattern_extend_ws_bytes(int n_heads, int S) {
    if (n_heads <= 0 || S <= 0) return 0;
    const size_t nqb = (static_cast<size_t>(S) + kTile - 1) / kTile;
    const size_t items = static_cast<size_t>(n_heads) * nqb;
    return align_up(sizeof(Totals)) + align_up(sizeof(int32_t) * 2 * n_heads) +
           align_up(sizeof(int32_t) * 2 * (n_heads + 1)) + align_up(sizeof(int32_t) * items) +
           align_up(sizeof(int32_t) * (items + 1)) +
           align_up(sizeof(int32_t) * static_cast<size_t>(n_heads) * static_cast<size_t>(S)) + 256;
}

namespace {

int extend_impl(int n_heads, const int32_t *diag_ptr, const int32_t *diag_offsets, const int32_t *vert_ptr,
                const int32_t *vert_cols, const uint32_t *true_mask, int L, int S, ssa_plan_sizes *sizes,
                const ssa_plan *plan, void *ws, size_t ws_bytes, int32_t *dev_status, void *stream) {
    SSA_CHECK_ARG(diag_ptr && diag_offsets && vert_ptr && vert_cols && ws,
                  "sparse_pattern_extend: null pointer argument");
    SSA_CHECK_ARG(n_heads >= 1 && S >= 1, "sparse_pattern_extend: n_heads and S must be >= 1");
    const int nqb = (S + kTile - 1) / kTile;
    SSA_CHECK_ARG(static_cast<int64_t>(n_heads) * nqb < (1 << 30),
                  "sparse_pattern_extend: n_heads * ceil(S/128) too large");
    const size_t need = sparse_pattern_extend_ws_bytes(n_heads, S);
    if (ws_bytes < need) {
        set_error("sparse_pattern_extend: workspace %zu bytes < required %zu", ws_bytes, need);
        return SSA_ERR_CAPACITY;
    }
    SSA_CHECK_ARG(aligned16(ws), "sparse_pattern_extend: ws must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    char *w = static_cast<char *>(ws);
    PlanParams p{};
    p.H = n_heads;
    p.S = S;
    p.nqb = nqb;
    p.dptr = diag_ptr;
    p.doff = diag_offsets;
    p.vptr = vert_ptr;
    p.vcol = vert_cols;
    p.totals = reinterpret_cast<Totals *>(w);
    w += align_up(sizeof(Totals));
    p.ws_status = &p.totals->status;
    p.ext_counts = reinterpret_cast<int32_t *>(w);
    w += align_up(sizeof(int32_t) * 2 * n_heads);
    p.ext_scan = reinterpret_cast<int32_t *>(w);
    w += align_up(sizeof(int32_t) * 2 * (n_heads + 1));
    p.tile_counts = reinterpret_cast<int32_t *>(w);
    w += align_up(sizeof(int32_t) * n_heads * nqb);
    p.tile_pos = reinterpret_cast<int32_t *>(w);
    w += align_up(sizeof(int32_t) * (n_heads * nqb + 1));
    p.run0 = reinterpret_cast<int32_t *>(w);
    p.dev_status = dev_status;

    const int items = n_heads * nqb;
    const unsigned tile_grid = static_cast<unsigned>((items + 3) / 4);
    int slots = 0;
    if (true_mask) {
        p.tmask = true_mask;
        p.L = L;
        p.bw = (L + 31) / 32;
        p.nL = (min(L, S) + kTile - 1) / kTile;
        slots = p.nL * (p.nL + 1) / 2;
        p.slots = slots;
    }
    SSA_CUDA_TRY(cudaMemsetAsync(p.totals, 0, sizeof(Totals), s));

    if (plan == nullptr) {
        SSA_CHECK_ARG(sizes, "sparse_pattern_extend: sizes must not be NULL in the sizing pass");
        validate_lists_kernel<<<n_heads, 128, 0, s>>>(p);
        SSA_LAUNCH_CHECK();
        run_start_kernel<<<n_heads, kScanThreads, 0, s>>>(p);
        SSA_LAUNCH_CHECK();
        plan_tiles_kernel<false><<<tile_grid, 128, 0, s>>>(p);
        SSA_LAUNCH_CHECK();
        exclusive_scan_kernel<<<1, kScanThreads, 0, s>>>(p.tile_counts, items, 1, 0, p.tile_pos,
                                                         &p.totals->n_tiles);
        SSA_LAUNCH_CHECK();
        plan_totals_kernel<<<1, 1024, 0, s>>>(p);
        SSA_LAUNCH_CHECK();
        Totals host{};
        SSA_CUDA_TRY(cudaMemcpyAsync(&host, p.totals, sizeof(Totals), cudaMemcpyDeviceToHost, s));
        SSA_CUDA_TRY(cudaStreamSynchronize(s));
        sizes->n_heads = n_heads;
        sizes->S = S;
        sizes->nqb = nqb;
        sizes->n_diag = host.n_diag;
        sizes->n_vert = host.n_vert;
        sizes->max_vert = host.max_vert;
        sizes->n_tiles = host.n_tiles;
        sizes->bitmap_slots = slots;
        if (host.status != 0) {
            set_error("sparse_pattern_extend: a pattern list is not strictly ascending and >= 0");
            return SSA_ERR_INVALID;
        }
        if (host.n_tiles > INT32_MAX) {
            set_error("sparse_pattern_extend: %lld tiles exceed the int32 tile offsets of a plan",
                      static_cast<long long>(host.n_tiles));
            return SSA_ERR_CAPACITY;
        }
        return SSA_OK;
    }

    SSA_CHECK_ARG(plan->n_heads == n_heads && plan->S == S && plan->nqb == nqb,
                  "sparse_pattern_extend: plan header (n_heads=%d S=%d nqb=%d) does not match "
                  "(%d, %d, %d)",
                  plan->n_heads, plan->S, plan->nqb, n_heads, S, nqb);
    SSA_CHECK_ARG(plan->ext_diag_ptr && plan->ext_diag_offsets && plan->ext_vert_ptr &&
                      plan->ext_vert_cols && plan->tile_ptr && plan->tile_key0 &&
                      plan->tile_dmask && plan->tile_cmask && plan->tile_flags &&
                      plan->stripe_cnt,
                  "sparse_pattern_extend: null plan array");
    SSA_CHECK_ARG(plan->n_tiles >= 0, "sparse_pattern_extend: negative tile capacity");
    if (true_mask) {
        SSA_CHECK_ARG(plan->tile_bits && plan->bitmap_slots == slots && aligned16(plan->tile_bits),
                      "sparse_pattern_extend_case2: plan needs tile_bits (16-byte aligned) for %d bitmap "
                      "slots per head",
                      slots);
        p.tile_bits = plan->tile_bits;
    }
    SSA_CHECK_ARG(plan->n_diag >= 0 && plan->n_vert >= 0 && plan->max_vert >= 0,
                  "sparse_pattern_extend: negative list capacity in the plan");
    p.tile_ptr = plan->tile_ptr;
    p.capacity = plan->n_tiles;
    p.cap_diag = plan->n_diag;
    p.cap_vert = plan->n_vert;
    p.cap_max_vert = plan->max_vert;
    p.tile_key0 = plan->tile_key0;
    p.tile_dmask = plan->tile_dmask;
    p.tile_cmask = plan->tile_cmask;
    p.tile_flags = plan->tile_flags;
    p.stripe_cnt = plan->stripe_cnt;
    p.ext_dptr = plan->ext_diag_ptr;
    p.ext_doff = plan->ext_diag_offsets;
    p.ext_vptr = plan->ext_vert_ptr;
    p.ext_vcol = plan->ext_vert_cols;

    // sizing of the new plan (workspace only), the capacity check, then the plan's writes
    validate_lists_kernel<<<n_heads, 128, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    exclusive_scan_kernel<<<1, kScanThreads, 0, s>>>(p.ext_counts, n_heads, 2, 0, p.ext_scan, nullptr);
    SSA_LAUNCH_CHECK();
    exclusive_scan_kernel<<<1, kScanThreads, 0, s>>>(p.ext_counts, n_heads, 2, 1,
                                                     p.ext_scan + (n_heads + 1), nullptr);
    SSA_LAUNCH_CHECK();
    run_start_kernel<<<n_heads, kScanThreads, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    plan_tiles_kernel<false><<<tile_grid, 128, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    exclusive_scan_kernel<<<1, kScanThreads, 0, s>>>(p.tile_counts, items, 1, 0, p.tile_pos, &p.totals->n_tiles);
    SSA_LAUNCH_CHECK();
    plan_check_kernel<<<1, 256, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    extend_copy_kernel<<<n_heads, 128, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    plan_tiles_kernel<true><<<tile_grid, 128, 0, s>>>(p);
    SSA_LAUNCH_CHECK();
    return SSA_OK;
}

}  // namespace

extern "C" int sparse_pattern_extend(int n_heads, const int32_t *diag_ptr,
                                     const int32_t *diag_offsets, const int32_t *vert_ptr,
                                     const int32_t *vert_cols, int S, ssa_plan_sizes *sizes,
                                     const ssa_plan *plan, void *ws, size_t ws_bytes,
                                     int32_t *dev_status, void *stream) {
    ssa::TraceRange trace_range("sparse_pattern_extend");
    return extend_impl(n_heads, diag_ptr, diag_offsets, vert_ptr, vert_cols, nullptr, 0, S, sizes, plan, ws,
                       ws_bytes, dev_status, stream);
}

extern "C" int sparse_pattern_extend_case2(int n_heads, const int32_t *diag_ptr,
                                           const int32_t *diag_offsets, const int32_t *vert_ptr,
                                           const int32_t *vert_cols, const uint32_t *true_mask, int L,
                                           int S, ssa_plan_sizes *sizes, const ssa_plan *plan, void *ws,
                                           size_t ws_bytes, int32_t *dev_status, void *stream) {
    ssa::TraceRange trace_range("sparse_pattern_extend_case2");
    SSA_CHECK_ARG(true_mask, "sparse_pattern_extend_case2: null true_mask");
    SSA_CHECK_ARG(L >= 1 && L <= 1024, "sparse_pattern_extend_case2: L must be in [1, 1024] (got %d)", L);
    SSA_CHECK_ARG((reinterpret_cast<uintptr_t>(true_mask) & 3u) == 0,
                  "sparse_pattern_extend_case2: true_mask must be 4-byte aligned");
    return extend_impl(n_heads, diag_ptr, diag_offsets, vert_ptr, vert_cols, true_mask, L, S, sizes, plan, ws,
                       ws_bytes, dev_status, stream);
}
