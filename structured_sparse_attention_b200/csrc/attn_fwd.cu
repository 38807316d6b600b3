// attn_fwd.cu -- causal sparse-attention prefill over the DAM extended mask.
//
// The mask is applied to QK^T / sqrt(d_k) before the softmax, so only the retained
// pairs take part (DAM review page: Referee Report summary; "Circularity Check"
// step 2; "What carries the argument": inference computes only the retained
// connections).  The page's own implementation forms the dense product and masks it
// (Referee Report major comment 1); here only the tiles that hold retained pairs are
// computed.
//
// Kernels
//   stripe_gather_kernel     K_C[h][k] = K[kv(h)][C_h[k]], V_C likewise, zero-padded to
//                            a multiple of 128 rows (the vertical-pattern columns of
//                            every head packed into dense tiles)
//   sparse_attn_fwd_kernel   one CTA per (head, 128-row query block):
//     warp 0     TMA producer: Q block once, then K/V tiles (band tiles from K/V at
//                the plan's key-tile index, then stripe tiles from K_C/V_C)
//     warp 1     allocates tensor memory; lane 0 issues tcgen05.mma:
//                S_j = Q K_j^T into a double-buffered TMEM S, O += P_j V_j with P read
//                from TMEM
//     warps 2-5  softmax: one thread per query row; tcgen05.ld S, element mask from the
//                plan (FULL tiles skip it), online max/sum in fp32 (log2 domain), P as
//                bf16 into TMEM, lazy O rescale (only when the max grows by > 2^8);
//                epilogue O / l -> bf16 and LSE
// Tensor memory (512 columns): S0 0..127, S1 128..255, P0 256..319, P1 320..383,
// O 384..384+d-1.  P has its own buffers so a QK^T never overwrites a P still being read.
// Barrier phases are tracked by tile index; every wait is on a barrier whose previous
// phase is known to have completed, so a parity never aliases two phases back.
// Every wait is bounded: on expiry the kernel records SSA_ERR_TIMEOUT, stops every role,
// drains its own copies and MMAs, frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace ssa {
namespace {

constexpr int kBM = SSA_BLOCK;
constexpr int kBN = SSA_BLOCK;
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 softmax (two halves per row)
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;
constexpr int kBoxBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr int64_t kDrainLimitNs = 1000000000LL;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale only if the max grows by > 256x

template <int D>
struct Cfg {
    static constexpr int NK = (D == 128) ? 3 : 4;  // K pipeline stages
    static constexpr int NV = (D == 128) ? 2 : 3;  // V pipeline stages
    static constexpr int BOXES = D / 64;
    static constexpr int TILE_BYTES = BOXES * kBoxBytes;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILE_BYTES;
    static constexpr int OFF_V = OFF_K + NK * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + NV * TILE_BYTES;
    // barriers + alignment slack; at least 120 KB so that a single CTA (and its 512
    // tensor-memory columns) occupies an SM
    static constexpr int SMEM_RAW = OFF_BAR + 4096 + 1024;
    static constexpr int SMEM_BYTES = SMEM_RAW > 120 * 1024 ? SMEM_RAW : 120 * 1024;
};

struct Barriers {
    uint64_t q_full;
    uint64_t k_full[4], v_full[4], k_empty[4], v_empty[4];
    uint64_t s_full[2], p_full[2], p_free[2];
    uint64_t epi_done;
    uint64_t mma_drain;
    uint64_t xchg[4][2];  // per TMEM lane quarter and tile parity: row-max exchange
    uint64_t lxchg[4];    // per quarter: final row-sum exchange
    uint32_t tmem_base;
    int abort;
    float red_max[2][2][128];  // [tile parity][column half][row]
    float red_l[2][128];       // [column half][row]
};
static_assert(sizeof(Barriers) <= 4096, "barrier block too large");

struct AttnParams {
    int S, H, Hkv, nqb, npad;
    const int32_t *tile_ptr;
    const int32_t *tile_kb;
    const uint64_t *tile_dmask;
    const uint64_t *tile_cmask;
    const uint32_t *tile_flags;
    const int32_t *stripe_cnt;
    const int32_t *vert_ptr;
    const int32_t *vert_cols;
    const int32_t *kv_map;
    float scale_log2;
    uint16_t *O;
    float *LSE;
    int32_t *status;
    int64_t wait_ns;
};

__device__ __forceinline__ int kv_head(const AttnParams &p, int h) {
    return p.kv_map ? __ldg(p.kv_map + h) : h / (p.H / p.Hkv);
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 "version 1" format).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 A/B, fp32 accumulate, A K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------------------------
// Stripe gather
// ---------------------------------------------------------------------------------

template <int D>
__global__ void __launch_bounds__(256) stripe_gather_kernel(const uint16_t *__restrict__ K,
                                                            const uint16_t *__restrict__ V,
                                                            uint16_t *__restrict__ KC,
                                                            uint16_t *__restrict__ VC,
                                                            AttnParams p) {
    constexpr int VEC = D / 8;  // 16-byte vectors per row
    constexpr int ROWS = 256 / VEC;
    const int h = blockIdx.y;
    const int row = blockIdx.x * ROWS + threadIdx.x / VEC;
    const int v = threadIdx.x % VEC;
    if (row >= p.npad) return;
    const int g = kv_head(p, h);
    const int c0 = p.vert_ptr[h], nc = p.vert_ptr[h + 1] - c0;
    uint4 kk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (g < 0 || g >= p.Hkv) {
        if (threadIdx.x == 0) report(p.status, SSA_ERR_INVALID);
    } else if (row < nc) {
        const int c = __ldg(p.vert_cols + c0 + row);
        if (c >= 0 && c < p.S) {
            const size_t src = (static_cast<size_t>(g) * p.S + c) * D;
            kk = __ldg(reinterpret_cast<const uint4 *>(K + src) + v);
            vv = __ldg(reinterpret_cast<const uint4 *>(V + src) + v);
        } else {
            report(p.status, SSA_ERR_INVALID);
        }
    }
    const size_t dst = (static_cast<size_t>(h) * p.npad + row) * D;
    reinterpret_cast<uint4 *>(KC + dst)[v] = kk;
    reinterpret_cast<uint4 *>(VC + dst)[v] = vv;
}

// ---------------------------------------------------------------------------------
// Attention forward
// ---------------------------------------------------------------------------------

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV,
                           const __grid_constant__ CUtensorMap tmKC,
                           const __grid_constant__ CUtensorMap tmVC, const AttnParams p) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    Barriers *bar = reinterpret_cast<Barriers *>(smem + C::OFF_BAR);
    volatile int *abort = &bar->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x;
    const int qb = p.nqb - 1 - item / p.H;  // heavy (late) query blocks first
    const int h = item % p.H;               // heads of one KV group side by side
    const int g = kv_head(p, h);
    const int tp0 = p.tile_ptr[h * p.nqb + qb];
    const int nb = p.tile_ptr[h * p.nqb + qb + 1] - tp0;
    const int sc = p.stripe_cnt[h * p.nqb + qb];
    int n = nb + (sc + kBN - 1) / kBN;
    if (g < 0 || g >= p.Hkv) {
        if (threadIdx.x == 0) report(p.status, SSA_ERR_INVALID);
        n = 0;
    }

    if (n == 0) {  // no retained key in this block: O = 0, LSE = -inf
        if (warp >= 2) {
            const int half = (warp - 2) >> 2;
            const int i = qb * kBM + 32 * (warp & 3) + lane;
            if (i < p.S) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.O + (static_cast<size_t>(h) * p.S + i) * D) +
                             half * (D / 16);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) dst[k] = make_uint4(0, 0, 0, 0);
                if (half == 0) p.LSE[static_cast<size_t>(h) * p.S + i] = -INFINITY;
            }
        }
        return;
    }

    if (threadIdx.x == 0) {
        mbar_init(&bar->q_full, 1);
        for (int s = 0; s < C::NK; ++s) {
            mbar_init(&bar->k_full[s], 1);
            mbar_init(&bar->k_empty[s], 1);
        }
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(&bar->v_full[s], 1);
            mbar_init(&bar->v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar->s_full[b], 1);
            mbar_init(&bar->p_full[b], kSoftmaxThreads);
            mbar_init(&bar->p_free[b], 1);
        }
        mbar_init(&bar->epi_done, kSoftmaxThreads);
        mbar_init(&bar->mma_drain, 1);
        for (int q = 0; q < 4; ++q) {
            mbar_init(&bar->xchg[q][0], 64);
            mbar_init(&bar->xchg[q][1], 64);
            mbar_init(&bar->lxchg[q], 64);
        }
        bar->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    const int64_t lim = p.wait_ns;

    if (warp == 0) {
        // ------------------------------ TMA producers -----------------------------
        // lane 0 streams Q then the K tiles, lane 1 the V tiles, each with its own ring
        if (lane < 2) {
            const bool is_k = (lane == 0);
            const int NSTG = is_k ? C::NK : C::NV;
            uint64_t *full = is_k ? bar->k_full : bar->v_full;
            uint64_t *empty = is_k ? bar->k_empty : bar->v_empty;
            uint8_t *ring = smem + (is_k ? C::OFF_K : C::OFF_V);
            const CUtensorMap *band_map = is_k ? &tmK : &tmV;
            const CUtensorMap *stripe_map = is_k ? &tmKC : &tmVC;
            prefetch_tmap(band_map);
            if (is_k) {
                prefetch_tmap(&tmQ);
                uint8_t *sQ = smem + C::OFF_Q;
                mbar_arrive_expect_tx(&bar->q_full, C::TILE_BYTES);
                for (int b = 0; b < C::BOXES; ++b)
                    tma_load_3d(sQ + b * kBoxBytes, &tmQ, &bar->q_full, 64 * b, qb * kBM, h);
            }
            int issued = 0;
            bool ok = true;
            int kb_next = (nb > 0) ? __ldg(p.tile_kb + tp0) : 0;
            for (int j = 0; j < n; ++j) {
                const int s = j % NSTG;
                const int kb = kb_next;
                if (j + 1 < nb) kb_next = __ldg(p.tile_kb + tp0 + j + 1);  // overlaps the wait
                if (j >= NSTG && !mbar_wait(&empty[s], ((j / NSTG) - 1) & 1, lim, abort)) {
                    ok = false;
                    break;
                }
                const bool band = j < nb;
                const CUtensorMap *map = band ? band_map : stripe_map;
                const int y = band ? kb * kBN : (j - nb) * kBN;
                const int z = band ? g : h;
                uint8_t *dst = ring + s * C::TILE_BYTES;
                mbar_arrive_expect_tx(&full[s], C::TILE_BYTES);
                for (int b = 0; b < C::BOXES; ++b)
                    tma_load_3d(dst + b * kBoxBytes, map, &full[s], 64 * b, y, z);
                issued = j + 1;
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            // Drain: never leave the CTA with a copy still writing shared memory.
            if (is_k) mbar_wait(&bar->q_full, 0, kDrainLimitNs, nullptr);
            for (int j = (issued > NSTG ? issued - NSTG : 0); j < issued; ++j)
                mbar_wait(&full[j % NSTG], (j / NSTG) & 1, kDrainLimitNs, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            constexpr uint32_t IDESC_QK = idesc_bf16(kBM, kBN, false);
            constexpr uint32_t IDESC_PV = idesc_bf16(kBM, D, true);
            const uint32_t sQ = smem_u32(smem + C::OFF_Q);
            bool ok = mbar_wait(&bar->q_full, 0, lim, abort);
            auto issue_pv = [&](int jj) -> bool {
                const int b = jj & 1, s = jj % C::NV;
                if (!mbar_wait(&bar->p_full[b], (jj >> 1) & 1, lim, abort)) return false;
                if (!mbar_wait(&bar->v_full[s], (jj / C::NV) & 1, lim, abort)) return false;
                tc_fence_after();
                const uint32_t sV = smem_u32(smem + C::OFF_V + s * C::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    // B = V tile, MN-major: 16 keys per step (2 x 8-row groups of 128 B)
                    const uint64_t bd = sdesc(sV + kk * 2048, kBoxBytes, 1024);
                    umma_ts(tmem + kColO, tmem + kColP + 64 * b + 8 * kk, bd, IDESC_PV,
                            (jj > 0 || kk > 0) ? 1u : 0u);
                }
                // p_free[b] completes once per PV that read P[b]: PV_b, PV_{b+2}, ... It
                // doubles as "O includes tile jj" (see the softmax waits).
                umma_commit(&bar->p_free[b]);
                umma_commit(&bar->v_empty[s]);
                return true;
            };
            for (int j = 0; j < n && ok; ++j) {
                const int s = j % C::NK, b = j & 1;
                if (!mbar_wait(&bar->k_full[s], (j / C::NK) & 1, lim, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sK = smem_u32(smem + C::OFF_K + s * C::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // A = Q, B = K tile, both K-major: 16 elements = 32 B per step
                    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                    umma_ss(tmem + kColS + 128 * b, sdesc(sQ + off, 16, 1024),
                            sdesc(sK + off, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bar->s_full[b]);
                umma_commit(&bar->k_empty[s]);
                if (j >= 1 && !issue_pv(j - 1)) ok = false;
            }
            if (ok && !issue_pv(n - 1)) ok = false;
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            umma_commit(&bar->mma_drain);  // completes once every issued MMA is done
        }
        __syncwarp();
        // Free tensor memory after the epilogue has read O and every MMA has finished.
        if (lane == 0) {
            mbar_wait(&bar->epi_done, 0, kDrainLimitNs, nullptr);
            mbar_wait(&bar->mma_drain, 0, kDrainLimitNs, nullptr);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    } else {
        // ------------------------------ softmax / epilogue ------------------------
        // Two threads per query row: warps 2-5 take key columns 0..63 of every tile,
        // warps 6-9 columns 64..127 (and the matching halves of O).  The row max of each
        // tile is exchanged through shared memory so both halves scale by the same
        // reference; each half keeps its own partial row sum until the epilogue.
        const int half = (warp - 2) >> 2;
        const int quarter = warp & 3;  // TMEM lane quarter this warp may access
        const int il = 32 * quarter + lane;
        const int i = qb * kBM + il;
        const bool row_ok = i < p.S;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
        const uint32_t col_s = kColS + 64 * half;     // + 128 * b: this half's S columns
        const uint32_t col_p = kColP + 32 * half;     // + 64 * b: this half's packed P columns
        const uint32_t col_o = kColO + (D / 2) * half; // this half's O columns
        const float sl2 = p.scale_log2;
        const int32_t *Ch = p.vert_cols + p.vert_ptr[h];
        const int nC = p.vert_ptr[h + 1] - p.vert_ptr[h];
        const int n_i = row_ok ? lower_bound_i32(Ch, nC, i + 1) : 0;  // columns c <= i

        // This half's 64-bit row mask of tile j (bit k = key column 64 * half + k).
        // Band tiles: local diagonal bits of the plan minus excluded columns; stripe
        // tiles: the first n_i - 128 * (j - nb) gathered columns.
        uint32_t m_flags = 0;
        uint64_t m_dm[4] = {0, 0, 0, 0}, m_cm[2] = {0, 0};
        auto fetch_meta = [&](int j) {  // raw plan data of band tile j (loads only)
            if (j < nb) {
                const size_t t = static_cast<size_t>(tp0 + j);
                m_flags = __ldg(p.tile_flags + t);
                const uint64_t *dmp = p.tile_dmask + 4 * t;
                m_dm[0] = __ldg(dmp);
                m_dm[1] = __ldg(dmp + 1);
                m_dm[2] = __ldg(dmp + 2);
                m_dm[3] = __ldg(dmp + 3);
                m_cm[0] = __ldg(p.tile_cmask + 2 * t + half);
            }
        };
        auto make_mask = [&](int j, bool &full, uint64_t &bits) {
            if (j < nb) {
                full = (m_flags & 1u) != 0;
                uint64_t lo, hi;
                row_diag_mask(m_dm, il, lo, hi);
                bits = (half ? hi : lo) & ~m_cm[0];
                if (!row_ok) bits = 0;
            } else {
                const int lim_k = n_i - (j - nb) * kBN - 64 * half;  // active iff k < lim_k
                full = lim_k >= 64;
                bits = lim_k >= 64 ? ~0ull : (lim_k <= 0 ? 0ull : (1ull << lim_k) - 1ull);
            }
        };
        bool cur_full = false;
        uint64_t cur_bits = 0;
        fetch_meta(0);
        make_mask(0, cur_full, cur_bits);
        fetch_meta(1);

        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int j = 0; j < n && ok; ++j) {
            const int b = j & 1;
            // tcgen05.ld is warp-collective: the whole warp proceeds or stops together
            if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full[b], (j >> 1) & 1, lim, abort))) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[64];
            {
                uint32_t r[64];
                tmem_ld32(tmem + lane_off + col_s + 128 * b, r);
                tmem_ld32(tmem + lane_off + col_s + 128 * b + 32, r + 32);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 64; ++k) sv[k] = __uint_as_float(r[k]);
            }
            // mask of the next tile from the metadata fetched one tile ahead
            bool nxt_full = false;
            uint64_t nxt_bits = 0;
            if (j + 1 < n) make_mask(j + 1, nxt_full, nxt_bits);
            if (j + 2 < n) fetch_meta(j + 2);

            if (!__all_sync(0xffffffffu, cur_full)) {
#pragma unroll
                for (int k = 0; k < 64; ++k)
                    if (!((cur_bits >> k) & 1ull)) sv[k] = -INFINITY;
            }
            float mx[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mx[c] = sv[c];
#pragma unroll
            for (int k = 8; k < 64; ++k) mx[k & 7] = fmaxf(mx[k & 7], sv[k]);
            float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
            // exchange the half-row maxima with the partner thread of the same row
            bar->red_max[b][half][il] = mt;
            mbar_arrive(&bar->xchg[quarter][b]);
            if (!__all_sync(0xffffffffu, mbar_wait(&bar->xchg[quarter][b], (j >> 1) & 1, lim, abort))) {
                ok = false;
                break;
            }
            mt = fmaxf(mt, bar->red_max[b][half ^ 1][il]);
            const float m_new = fmaxf(m_run, mt * sl2);
            // lazy rescale: keep a stale max unless the row max grew by more than 2^8
            const bool grow = (m_new != -INFINITY) &&
                              (m_run == -INFINITY || m_new > m_run + kRescaleThreshold);
            const bool need_o = grow && (m_run != -INFINITY);
            float factor = 1.0f;
            if (grow) {
                factor = (m_run == -INFINITY) ? 0.0f : ex2_approx(m_run - m_new);
                l_run *= factor;
                m_run = m_new;
            }
            if (__any_sync(0xffffffffu, need_o)) {  // warp-uniform: O is read warp-collectively
                // O must include P_{j-1} V_{j-1} before it is rescaled.  PV_{j-1} is the
                // ((j-1) >> 1)-th completion of p_free[(j-1) & 1]; PV_{j-3}, the phase before
                // it, completed before P_{j-1} was written, so the parity cannot alias.
                if (!__all_sync(0xffffffffu, mbar_wait(&bar->p_free[(j - 1) & 1], ((j - 1) >> 1) & 1, lim, abort))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float f = need_o ? factor : 1.0f;
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + col_o + 32 * c, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * f);
                    tmem_st32(tmem + lane_off + col_o + 32 * c, r);
                }
            }
            const float mref = (m_run == -INFINITY) ? 0.0f : m_run;
            // P[b] may still be read by the MMA of tile j - 2
            if (j >= 2 && !__all_sync(0xffffffffu,
                                      mbar_wait(&bar->p_free[b], ((j >> 1) - 1) & 1, lim, abort))) {
                ok = false;
                break;
            }
            float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint32_t r[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float p0 = ex2_approx(fmaf(sv[2 * k], sl2, -mref));
                const float p1 = ex2_approx(fmaf(sv[2 * k + 1], sl2, -mref));
                ls[(2 * k) & 7] += p0;
                ls[(2 * k + 1) & 7] += p1;
                const __nv_bfloat162 pk = __floats2bfloat162_rn(p0, p1);
                r[k] = *reinterpret_cast<const uint32_t *>(&pk);
            }
            tmem_st32(tmem + lane_off + col_p + 64 * b, r);
            l_run += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar->p_full[b]);
            cur_full = nxt_full;
            cur_bits = nxt_bits;
        }
        if (ok) {
            // row sum = both halves' partial sums
            bar->red_l[half][il] = l_run;
            mbar_arrive(&bar->lxchg[quarter]);
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->lxchg[quarter], 0, lim, abort));
        }
        if (ok) {
            // O complete: PV_{n-1} done (the phase before it, PV_{n-3}, was awaited before
            // P_{n-1} was written)
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->p_free[(n - 1) & 1], ((n - 1) >> 1) & 1, lim, abort));
        }
        if (ok) {
            tc_fence_after();
            const float l_tot = l_run + bar->red_l[half ^ 1][il];
            const float inv = (l_tot > 0.0f) ? 1.0f / l_tot : 0.0f;
            uint4 *dst = reinterpret_cast<uint4 *>(p.O + (static_cast<size_t>(h) * p.S + (row_ok ? i : 0)) * D) +
                         half * (D / 16);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_off + col_o + 32 * c, r);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 v2 = __floats2bfloat162_rn(
                                __uint_as_float(r[8 * k + 2 * e]) * inv,
                                __uint_as_float(r[8 * k + 2 * e + 1]) * inv);
                            w[e] = *reinterpret_cast<const uint32_t *>(&v2);
                        }
                        dst[4 * c + k] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            if (row_ok && half == 0)
                p.LSE[static_cast<size_t>(h) * p.S + i] =
                    (l_tot > 0.0f) ? (m_run + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
        } else {
            report(p.status, SSA_ERR_TIMEOUT);
            *abort = 1;
        }
        tc_fence_before();
        mbar_arrive(&bar->epi_done);
    }
}

// ---------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 3-D map over bf16 [heads][rows][d]; box = 64 columns x 128 rows x 1, 128-byte swizzle.
int make_map(CUtensorMap *m, const void *base, int d, int rows, int heads) {
    auto enc = get_encode_fn();
    if (!enc) {
        set_error("cuTensorMapEncodeTiled is unavailable");
        return SSA_ERR_CUDA;
    }
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(heads)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                             static_cast<cuuint64_t>(rows) * d * 2};
    cuuint32_t box[3] = {64, kBM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) for rows=%d heads=%d d=%d", static_cast<int>(r),
                  rows, heads, d);
        return SSA_ERR_CUDA;
    }
    return SSA_OK;
}

template <int D>
int launch(const void *Q, const void *K, const void *V, uint16_t *KC, uint16_t *VC, AttnParams &p,
           cudaStream_t s) {
    using C = Cfg<D>;
    if (p.npad > 0) {
        constexpr int ROWS = 256 / (D / 8);
        dim3 grid((p.npad + ROWS - 1) / ROWS, p.H);
        stripe_gather_kernel<D><<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(K),
                                                     static_cast<const uint16_t *>(V), KC, VC, p);
        SSA_LAUNCH_CHECK();
    }
    CUtensorMap mQ, mK, mV, mKC, mVC;
    int rc;
    if ((rc = make_map(&mQ, Q, D, p.S, p.H)) != SSA_OK) return rc;
    if ((rc = make_map(&mK, K, D, p.S, p.Hkv)) != SSA_OK) return rc;
    if ((rc = make_map(&mV, V, D, p.S, p.Hkv)) != SSA_OK) return rc;
    if (p.npad > 0) {
        if ((rc = make_map(&mKC, KC, D, p.npad, p.H)) != SSA_OK) return rc;
        if ((rc = make_map(&mVC, VC, D, p.npad, p.H)) != SSA_OK) return rc;
    } else {
        mKC = mK;  // never read: no stripe tiles without columns
        mVC = mV;
    }
    SSA_CUDA_TRY(cudaFuncSetAttribute(sparse_attn_fwd_kernel<D>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    const unsigned grid = static_cast<unsigned>(p.H) * static_cast<unsigned>(p.nqb);
    sparse_attn_fwd_kernel<D><<<grid, kThreads, C::SMEM_BYTES, s>>>(mQ, mK, mV, mKC, mVC, p);
    SSA_LAUNCH_CHECK();
    return SSA_OK;
}

size_t round_up128(size_t x) { return (x + 127) / 128 * 128; }

}  // namespace
}  // namespace ssa

using namespace ssa;

extern "C" size_t sparse_attn_fwd_ws_bytes(int n_heads, int max_vert, int d) {
    if (n_heads <= 0 || max_vert < 0 || d <= 0) return 0;
    return 2 * static_cast<size_t>(n_heads) * round_up128(static_cast<size_t>(max_vert)) * d *
           sizeof(uint16_t);
}

extern "C" int sparse_attn_fwd(const void *Q, const void *K, const void *V, int H_q, int H_kv,
                               int S, int d, const ssa_plan *plan, const int32_t *kv_map,
                               float scale, void *O, float *LSE, void *ws, size_t ws_bytes,
                               int32_t *dev_status, void *stream) {
    SSA_CHECK_ARG(Q && K && V && O && LSE && plan, "sparse_attn_fwd: null pointer argument");
    if (d != 64 && d != 128) {
        set_error("sparse_attn_fwd: head dimension must be 64 or 128 (got %d)", d);
        return SSA_ERR_UNSUPPORTED;
    }
    SSA_CHECK_ARG(H_q >= 1 && H_kv >= 1 && S >= 1, "sparse_attn_fwd: H_q, H_kv, S must be >= 1");
    SSA_CHECK_ARG(kv_map || H_q % H_kv == 0,
                  "sparse_attn_fwd: H_q (%d) must be a multiple of H_kv (%d) without kv_map", H_q,
                  H_kv);
    SSA_CHECK_ARG(plan->S == S && plan->n_heads == H_q && plan->nqb == (S + kBM - 1) / kBM,
                  "sparse_attn_fwd: plan (S=%d heads=%d) does not match S=%d H_q=%d", plan->S,
                  plan->n_heads, S, H_q);
    SSA_CHECK_ARG(plan->tile_ptr && plan->tile_kb && plan->tile_dmask && plan->tile_cmask &&
                      plan->tile_flags && plan->stripe_cnt && plan->ext_vert_ptr &&
                      plan->ext_vert_cols,
                  "sparse_attn_fwd: null plan array");
    SSA_CHECK_ARG(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O),
                  "sparse_attn_fwd: Q, K, V and O must be 16-byte aligned");
    SSA_CHECK_ARG(scale > 0.0f && scale < 1e30f, "sparse_attn_fwd: scale must be positive and finite");
    SSA_CHECK_ARG(static_cast<int64_t>(H_q) * ((S + kBM - 1) / kBM) < (1LL << 31),
                  "sparse_attn_fwd: too many query blocks");
    const size_t need = sparse_attn_fwd_ws_bytes(H_q, plan->max_vert, d);
    if (need > 0) {
        SSA_CHECK_ARG(ws && aligned16(ws), "sparse_attn_fwd: ws must be a 16-byte aligned buffer");
        if (ws_bytes < need) {
            set_error("sparse_attn_fwd: workspace %zu bytes < required %zu", ws_bytes, need);
            return SSA_ERR_CAPACITY;
        }
    }
    AttnParams p{};
    p.S = S;
    p.H = H_q;
    p.Hkv = H_kv;
    p.nqb = plan->nqb;
    p.npad = static_cast<int>(round_up128(static_cast<size_t>(plan->max_vert)));
    p.tile_ptr = plan->tile_ptr;
    p.tile_kb = plan->tile_kb;
    p.tile_dmask = plan->tile_dmask;
    p.tile_cmask = plan->tile_cmask;
    p.tile_flags = plan->tile_flags;
    p.stripe_cnt = plan->stripe_cnt;
    p.vert_ptr = plan->ext_vert_ptr;
    p.vert_cols = plan->ext_vert_cols;
    p.kv_map = kv_map;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.O = static_cast<uint16_t *>(O);
    p.LSE = LSE;
    p.status = dev_status;
    p.wait_ns = wait_limit_ns();
    uint16_t *KC = static_cast<uint16_t *>(ws);
    uint16_t *VC = KC ? KC + static_cast<size_t>(H_q) * p.npad * d : nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d == 64 ? launch<64>(Q, K, V, KC, VC, p, s) : launch<128>(Q, K, V, KC, VC, p, s);
}
