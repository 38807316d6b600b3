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
//   sparse_attn_fwd_kernel   persistent: one CTA per SM takes work items (head,
//                            128-row query block) from a global counter, heaviest
//                            query blocks first.  Roles:
//     warp 8 lane 0  scheduler + TMA producer of Q and K tiles (band tiles from K at
//                    the plan's key-tile index, then stripe tiles from K_C)
//     warp 8 lane 1  TMA producer of V tiles
//     warp 9         allocates tensor memory; lane 0 issues tcgen05.mma:
//                    S_t = Q K_t^T into a double-buffered TMEM S, O += P_t V_t with P
//                    read from TMEM.  QK^T of tile t+2 is issued as soon as the softmax
//                    has read S_t, ahead of PV of tile t.
//     warps 0-7      softmax, two threads per query row (key columns 0-63 / 64-127 and
//                    the matching O halves), software-pipelined one tile ahead:
//                    tcgen05.ld S, element mask from the plan (FULL tiles skip it), row
//                    max exchanged through shared memory at a named barrier, online
//                    max/sum in fp32 (log2 domain, packed f32x2 arithmetic), P as bf16
//                    into TMEM, lazy O rescale (only when the max grows by > 2^8);
//                    epilogue O / l -> bf16 and LSE.
// Tensor memory (512 columns): S0 0..127, S1 128..255, P0 256..319, P1 320..383,
// O 384..384+d-1.  P has its own buffers so a QK^T never overwrites a P being read.
//
// Barrier phases follow global counters (tiles t across items, items m, non-empty
// items e).  Every wait is on a barrier whose previous phase is known to be complete,
// so a parity never aliases two phases back.  Every wait is bounded: on expiry the
// kernel records SSA_ERR_TIMEOUT, stops every role, drains its own copies and MMAs,
// frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace ssa {
namespace {

constexpr int kBM = SSA_BLOCK;
constexpr int kBN = SSA_BLOCK;
// Warps 0-7 softmax (two warpgroups), warp 8 TMA producers, warp 9 MMA issuer, warps
// 10-11 idle.  Registers are rebalanced with setmaxnreg: the launch gives every thread
// kLaunchRegs; the TMA/MMA warpgroup drops to kCtrlRegs and the softmax warpgroups
// rise to kSoftmaxRegs, which together use exactly the launch allocation.
constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;
constexpr int kSoftmaxWarps = 8;
constexpr int kWarpTma = 8, kWarpMma = 9;
constexpr int kLaunchRegs = 168, kCtrlRegs = 56, kSoftmaxRegs = 224;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kCtrlRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kRing = 4;  // work-item descriptors in flight
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;
constexpr int kBoxBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr int64_t kDrainLimitNs = 1000000000LL;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale only if the max grows by > 256x
constexpr size_t kCounterBytes = 256;     // work counter at the start of the workspace

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

struct ItemDesc {
    int h, qb, g, tp0, nb, n, stripe_lo;  // n < 0 marks the end of the work
};

struct Shared {
    uint64_t item_full[kRing], item_empty[kRing];
    uint64_t q_full, q_empty;
    uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
    uint64_t s_full[2], s_free[2], p_full[2], p_free[2];
    uint64_t o_free;
    uint64_t mma_drain, softmax_done;
    ItemDesc items[kRing];
    uint32_t tmem_base;
    int abort;
    float red_max[2][2][128];  // [tile parity][column half][row]
    float red_l[2][128];       // [column half][row]
};
static_assert(sizeof(Shared) <= 4096, "barrier block too large");

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
    int *work_counter;
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
// Attention forward (persistent)
// ---------------------------------------------------------------------------------

// Work item idx -> descriptor.  Items run from the last query block down (later
// blocks hold more tiles under causal patterns) with the heads of one block side by
// side, so heads of a KV group read the same key tiles close together in time.
__device__ ItemDesc make_item(const AttnParams &p, int idx) {
    ItemDesc d;
    d.qb = p.nqb - 1 - idx / p.H;
    d.h = idx % p.H;
    d.g = kv_head(p, d.h);
    const int it = d.h * p.nqb + d.qb;
    d.tp0 = p.tile_ptr[it];
    d.nb = p.tile_ptr[it + 1] - d.tp0;
    const int sc = p.stripe_cnt[it];
    d.stripe_lo = d.qb > 0 ? p.stripe_cnt[it - 1] : 0;
    d.n = d.nb + (sc + kBN - 1) / kBN;
    if (d.g < 0 || d.g >= p.Hkv) {
        report(p.status, SSA_ERR_INVALID);
        d.n = 0;  // still writes O = 0, LSE = -inf
    }
    return d;
}

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
    Shared *sh = reinterpret_cast<Shared *>(smem + C::OFF_BAR);
    volatile int *abort = &sh->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = p.H * p.nqb;

    if (threadIdx.x == 0) {
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&sh->item_full[r], 1);
            mbar_init(&sh->item_empty[r], 2 + kSoftmaxWarps);  // V lane, MMA, softmax warps
        }
        mbar_init(&sh->q_full, 1);
        mbar_init(&sh->q_empty, 1);
        for (int s = 0; s < C::NK; ++s) {
            mbar_init(&sh->k_full[s], 1);
            mbar_init(&sh->k_empty[s], 1);
        }
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(&sh->v_full[s], 1);
            mbar_init(&sh->v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh->s_full[b], 1);
            mbar_init(&sh->s_free[b], kSoftmaxThreads);
            mbar_init(&sh->p_full[b], kSoftmaxThreads);
            mbar_init(&sh->p_free[b], 1);
        }
        mbar_init(&sh->o_free, kSoftmaxThreads);
        mbar_init(&sh->mma_drain, 1);
        mbar_init(&sh->softmax_done, kSoftmaxThreads);
        sh->abort = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&sh->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;
    const int64_t lim = p.wait_ns;
    if (warp >= kSoftmaxWarps) {
      // ------------------------- control warpgroup (warps 8-11) -------------------------
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
      if (warp == kWarpTma) {
        if (lane == 0) {
            // --------------------- scheduler + Q/K producer ---------------------
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmKC);
            bool ok = true;
            int m = 0, e = 0, t = 0;
            while (ok) {
                const int idx = atomicAdd(p.work_counter, 1);
                const int slot = m % kRing;
                if (m >= kRing && !mbar_wait(&sh->item_empty[slot], ((m / kRing) - 1) & 1, lim, abort)) {
                    ok = false;
                    break;
                }
                ItemDesc d;
                if (idx < n_items) {
                    d = make_item(p, idx);
                } else {
                    d.n = -1;
                }
                sh->items[slot] = d;
                mbar_arrive(&sh->item_full[slot]);  // release: the descriptor is visible
                ++m;
                if (d.n < 0) break;
                if (d.n == 0) continue;
                // Q block of this item, once the previous item's last QK^T is done
                if (e >= 1 && !mbar_wait(&sh->q_empty, (e - 1) & 1, lim, abort)) {
                    ok = false;
                    break;
                }
                uint8_t *sQ = smem + C::OFF_Q;
                mbar_arrive_expect_tx(&sh->q_full, C::TILE_BYTES);
                for (int b = 0; b < C::BOXES; ++b)
                    tma_load_3d(sQ + b * kBoxBytes, &tmQ, &sh->q_full, 64 * b, d.qb * kBM, d.h);
                ++e;
                int kb_next = d.nb > 0 ? __ldg(p.tile_kb + d.tp0) : 0;
                for (int j = 0; j < d.n; ++j, ++t) {
                    const int s = t % C::NK;
                    const int kb = kb_next;
                    if (j + 1 < d.nb) kb_next = __ldg(p.tile_kb + d.tp0 + j + 1);
                    if (t >= C::NK && !mbar_wait(&sh->k_empty[s], ((t / C::NK) - 1) & 1, lim, abort)) {
                        ok = false;
                        break;
                    }
                    const bool band = j < d.nb;
                    uint8_t *dst = smem + C::OFF_K + s * C::TILE_BYTES;
                    mbar_arrive_expect_tx(&sh->k_full[s], C::TILE_BYTES);
                    for (int b = 0; b < C::BOXES; ++b)
                        tma_load_3d(dst + b * kBoxBytes, band ? &tmK : &tmKC, &sh->k_full[s], 64 * b,
                                    band ? kb * kBN : (j - d.nb) * kBN, band ? d.g : d.h);
                }
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            // Drain: never leave the CTA with a copy still writing shared memory.
            if (e >= 1) mbar_wait(&sh->q_full, (e - 1) & 1, kDrainLimitNs, nullptr);
            for (int u = (t > C::NK ? t - C::NK : 0); u < t; ++u)
                mbar_wait(&sh->k_full[u % C::NK], (u / C::NK) & 1, kDrainLimitNs, nullptr);
        } else if (lane == 1) {
            // ----------------------------- V producer ----------------------------
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmVC);
            bool ok = true;
            int m = 0, t = 0;
            while (ok) {
                const int slot = m % kRing;
                if (!mbar_wait(&sh->item_full[slot], (m / kRing) & 1, lim, abort)) {
                    ok = false;
                    break;
                }
                const ItemDesc d = sh->items[slot];
                mbar_arrive(&sh->item_empty[slot]);
                ++m;
                if (d.n < 0) break;
                int kb_next = d.nb > 0 ? __ldg(p.tile_kb + d.tp0) : 0;
                for (int j = 0; j < d.n; ++j, ++t) {
                    const int s = t % C::NV;
                    const int kb = kb_next;
                    if (j + 1 < d.nb) kb_next = __ldg(p.tile_kb + d.tp0 + j + 1);
                    if (t >= C::NV && !mbar_wait(&sh->v_empty[s], ((t / C::NV) - 1) & 1, lim, abort)) {
                        ok = false;
                        break;
                    }
                    const bool band = j < d.nb;
                    uint8_t *dst = smem + C::OFF_V + s * C::TILE_BYTES;
                    mbar_arrive_expect_tx(&sh->v_full[s], C::TILE_BYTES);
                    for (int b = 0; b < C::BOXES; ++b)
                        tma_load_3d(dst + b * kBoxBytes, band ? &tmV : &tmVC, &sh->v_full[s], 64 * b,
                                    band ? kb * kBN : (j - d.nb) * kBN, band ? d.g : d.h);
                }
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            for (int u = (t > C::NV ? t - C::NV : 0); u < t; ++u)
                mbar_wait(&sh->v_full[u % C::NV], (u / C::NV) & 1, kDrainLimitNs, nullptr);
        }
      } else if (warp == kWarpMma) {
        // --------------------------------- MMA issuer ---------------------------------
        if (lane == 0) {
            constexpr uint32_t IDESC_QK = idesc_bf16(kBM, kBN, false);
            constexpr uint32_t IDESC_PV = idesc_bf16(kBM, D, true);
            const uint32_t sQ = smem_u32(smem + C::OFF_Q);
            bool ok = true;
            // Two cursors over the global tile sequence: QK^T (item mq, tile jq, global
            // tile tq) runs up to two tiles ahead of PV (item mp, tile jp, global tile tp).
            // eq / ep count non-empty items started by each cursor.  Readiness is polled
            // without blocking and a ready PV always goes first: the softmax warps (and
            // the epilogue) wait for PVs, never for a QK^T of a later tile.
            int mq = 0, jq = 0, tq = 0, eq = 0, nq = 0;
            int mp = 0, jp = 0, tp = 0, ep = 0;
            bool q_loaded = false, q_end = false;
            uint64_t t_progress = global_timer_ns();
            while (true) {
                bool progress = false;
                // QK cursor: load descriptors until a tile is available (never more than
                // kRing - 1 items ahead of the PV cursor, whose ring slot it would need)
                while (!q_end && !(q_loaded && jq < nq)) {
                    if (q_loaded) {
                        ++mq;
                        jq = 0;
                        q_loaded = false;
                    }
                    if (mq - mp >= kRing - 1) break;
                    if (!mbar_test(&sh->item_full[mq % kRing], (mq / kRing) & 1)) break;
                    nq = sh->items[mq % kRing].n;
                    q_loaded = true;
                    if (nq < 0) q_end = true;
                    progress = true;
                }
                // PV cursor: step over empty or finished items, releasing their slots
                bool pv_end = false;
                while (mp < mq || (q_loaded && mp == mq)) {
                    const int np = sh->items[mp % kRing].n;
                    if (np < 0) {
                        pv_end = true;
                        break;
                    }
                    if (jp < np) break;
                    mbar_arrive(&sh->item_empty[mp % kRing]);
                    ++mp;
                    jp = 0;
                    progress = true;
                }
                if (pv_end && tp == tq) break;  // every MMA issued
                if (tp < tq) {
                    // ---- PV of tile tp (item mp, tile jp) ----
                    const int b = tp & 1, s = tp % C::NV;
                    // the previous item's epilogue must have read O before PV overwrites it
                    const bool o_ok = !(jp == 0 && ep >= 1) || mbar_test(&sh->o_free, (ep - 1) & 1);
                    if (o_ok && mbar_test(&sh->p_full[b], (tp >> 1) & 1) &&
                        mbar_test(&sh->v_full[s], (tp / C::NV) & 1)) {
                        tc_fence_after();
                        const uint32_t sV = smem_u32(smem + C::OFF_V + s * C::TILE_BYTES);
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk) {
                            // B = V tile, MN-major: 16 keys per step (2 x 8-row groups of 128 B)
                            const uint64_t bd = sdesc(sV + kk * 2048, kBoxBytes, 1024);
                            umma_ts(tmem + kColO, tmem + kColP + 64 * b + 8 * kk, bd, IDESC_PV,
                                    (jp > 0 || kk > 0) ? 1u : 0u);
                        }
                        // p_free[b] completes once per PV that read P[b]: PV_b, PV_{b+2}, ...
                        // It doubles as "O includes tile tp" for the softmax warps.
                        umma_commit(&sh->p_free[b]);
                        umma_commit(&sh->v_empty[s]);
                        if (jp == 0) ++ep;
                        ++jp;
                        ++tp;
                        t_progress = global_timer_ns();
                        continue;
                    }
                }
                if (!q_end && q_loaded && jq < nq && tq <= tp + 2) {
                    // ---- QK^T of tile tq (item mq, tile jq) ----
                    const int s = tq % C::NK, b = tq & 1;
                    // S[b] is free once the softmax has read S_{tq-2}
                    if ((jq != 0 || mbar_test(&sh->q_full, eq & 1)) &&
                        mbar_test(&sh->k_full[s], (tq / C::NK) & 1) &&
                        (tq < 2 || mbar_test(&sh->s_free[b], ((tq - 2) >> 1) & 1))) {
                        tc_fence_after();
                        const uint32_t sK = smem_u32(smem + C::OFF_K + s * C::TILE_BYTES);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            // A = Q, B = K tile, both K-major: 16 elements = 32 B per step
                            const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                            umma_ss(tmem + kColS + 128 * b, sdesc(sQ + off, 16, 1024),
                                    sdesc(sK + off, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&sh->s_full[b]);
                        umma_commit(&sh->k_empty[s]);
                        if (jq == nq - 1) umma_commit(&sh->q_empty);  // Q of this item no longer read
                        if (jq == 0) ++eq;
                        ++jq;
                        ++tq;
                        t_progress = global_timer_ns();
                        continue;
                    }
                }
                if (progress) {
                    t_progress = global_timer_ns();
                    continue;
                }
                if (*abort || static_cast<int64_t>(global_timer_ns() - t_progress) >= lim) {
                    ok = false;
                    break;
                }
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            umma_commit(&sh->mma_drain);  // completes once every issued MMA is done
        }
        __syncwarp();
        // Free tensor memory after the softmax warps are done and every MMA has finished.
        if (lane == 0) {
            mbar_wait(&sh->softmax_done, 0, kDrainLimitNs, nullptr);
            mbar_wait(&sh->mma_drain, 0, kDrainLimitNs, nullptr);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // -------------------------------- softmax / epilogue -------------------------------
        // Two threads per query row: warps 0-3 take key columns 0..63 of every tile,
        // warps 4-7 columns 64..127 (and the matching halves of O).  The two warps of a
        // row quarter exchange each tile's half-row maxima through shared memory at a
        // named barrier, so both scale by the same reference; each keeps its own partial
        // row sum until the epilogue.  The loop is software-pipelined: while the exps of
        // tile j run (MUFU-bound), tile j+1 is loaded, masked and reduced.
        // A failed wait never leaves a warp early: it marks `good` false, raises the
        // abort flag and is carried into the next named-barrier reduction, where both
        // warps of the pair leave together.
        const int half = warp >> 2;
        const int quarter = warp & 3;  // TMEM lane quarter this warp may access
        const int bar_id = 1 + quarter;
        const int il = 32 * quarter + lane;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
        const uint32_t col_s = kColS + 64 * half;       // + 128 * b: this half's S columns
        const uint32_t col_p = kColP + 32 * half;       // + 64 * b: this half's packed P columns
        const uint32_t col_o = kColO + (D / 2) * half;  // this half's O columns
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        bool ok = true;
        bool good = true;  // sticky: false after any failed wait in this warp
        auto fail = [&]() {
            good = false;
            *abort = 1;
        };
        int m = 0, e = 0, t = 0;
        while (true) {
            const int slot = m % kRing;
            if (good && !__all_sync(0xffffffffu, mbar_wait(&sh->item_full[slot], (m / kRing) & 1, lim, abort)))
                fail();
            // both warps of the pair take every item (or leave) together
            if (!bar_and(bar_id, 64, good)) {
                ok = false;
                break;
            }
            const ItemDesc d = sh->items[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->item_empty[slot]);
            ++m;
            if (d.n < 0) break;
            const int i = d.qb * kBM + il;
            const bool row_ok = i < p.S;
            uint4 *orow = reinterpret_cast<uint4 *>(p.O + (static_cast<size_t>(d.h) * p.S + (row_ok ? i : 0)) * D) +
                          half * (D / 16);
            if (d.n == 0) {  // no retained key in this block: O = 0, LSE = -inf
                if (row_ok) {
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) orow[k] = make_uint4(0, 0, 0, 0);
                    if (half == 0) p.LSE[static_cast<size_t>(d.h) * p.S + i] = -INFINITY;
                }
                continue;
            }
            // stripe columns c <= i: between the counts of the previous and this block
            int n_i = 0;
            if (row_ok && d.n > d.nb) {
                const int32_t *Ch = p.vert_cols + p.vert_ptr[d.h];
                const int hi = p.stripe_cnt[d.h * p.nqb + d.qb];
                n_i = d.stripe_lo + lower_bound_i32(Ch + d.stripe_lo, hi - d.stripe_lo, i + 1);
            }

            // This half's 64-bit row mask of tile j (bit k = key column 64 * half + k).
            uint32_t m_flags = 0;
            uint64_t m_dm[4] = {0, 0, 0, 0}, m_cm = 0;
            auto fetch_meta = [&](int j) {  // raw plan data of band tile j (loads only)
                if (j < d.nb) {
                    const size_t tt = static_cast<size_t>(d.tp0 + j);
                    m_flags = __ldg(p.tile_flags + tt);
                    const uint64_t *dmp = p.tile_dmask + 4 * tt;
                    m_dm[0] = __ldg(dmp);
                    m_dm[1] = __ldg(dmp + 1);
                    m_dm[2] = __ldg(dmp + 2);
                    m_dm[3] = __ldg(dmp + 3);
                    m_cm = __ldg(p.tile_cmask + 2 * tt + half);
                }
            };
            auto make_mask = [&](int j, bool &full, uint64_t &bits) {
                if (j < d.nb) {
                    full = (m_flags & 1u) != 0;
                    uint64_t lo, hi;
                    row_diag_mask(m_dm, il, lo, hi);
                    bits = (half ? hi : lo) & ~m_cm;
                    if (!row_ok) bits = 0;
                } else {
                    const int lim_k = n_i - (j - d.nb) * kBN - 64 * half;  // active iff k < lim_k
                    full = lim_k >= 64;
                    bits = lim_k >= 64 ? ~0ull : (lim_k <= 0 ? 0ull : (1ull << lim_k) - 1ull);
                }
            };
            // S of global tile tt -> dst; releases S[tt & 1] for the QK^T of tile tt + 2
            auto load_s = [&](int tt, float(&dst)[64]) {
                const int bb = tt & 1;
                if (!good || !__all_sync(0xffffffffu, mbar_wait(&sh->s_full[bb], (tt >> 1) & 1, lim, abort))) {
                    fail();
                    return;
                }
                tc_fence_after();
                uint32_t r[64];
                tmem_ld32(tmem + lane_off + col_s + 128 * bb, r);
                tmem_ld32(tmem + lane_off + col_s + 128 * bb + 32, r + 32);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&sh->s_free[bb]);
#pragma unroll
                for (int k = 0; k < 64; ++k) dst[k] = __uint_as_float(r[k]);
            };
            auto apply_mask = [&](float(&v)[64], uint64_t bits) {
#pragma unroll
                for (int k = 0; k < 64; ++k)
                    if (!((bits >> k) & 1ull)) v[k] = -INFINITY;
            };
            auto half_max = [&](const float(&v)[64]) {
                float mx[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
                for (int k = 4; k < 64; k += 8) {
                    mx[0] = fmax3(mx[0], v[k], v[k + 1]);
                    mx[1] = fmax3(mx[1], v[k + 2], v[k + 3]);
                    mx[2] = fmax3(mx[2], v[k + 4], v[k + 5]);
                    mx[3] = fmax3(mx[3], v[k + 6], v[k + 7]);
                }
                return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            };
            // P = 2^(s * scale_log2 - mref) as packed bf16 pairs; returns the row-sum part
            auto exps = [&](const float(&v)[64], float mref, uint32_t(&pk)[32]) {
                const uint64_t nm2 = f2_pack(-mref, -mref);
                uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(v[2 * k], v[2 * k + 1]), sl2x2, nm2), x0, x1);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    acc[k & 3] = f2_add(acc[k & 3], f2_pack(p0, p1));
                    const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                    pk[k] = *reinterpret_cast<const uint32_t *>(&pb);
                }
                float a0, a1, a2, a3, a4, a5, a6, a7;
                f2_unpack(acc[0], a0, a1);
                f2_unpack(acc[1], a2, a3);
                f2_unpack(acc[2], a4, a5);
                f2_unpack(acc[3], a6, a7);
                return ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
            };

            // ---- prologue: first tile loaded, masked, its row max exchanged ----
            float sA[64], sB[64];
            bool nxt_full = false;
            uint64_t nxt_bits = 0;
            fetch_meta(0);
            make_mask(0, nxt_full, nxt_bits);
            fetch_meta(1);
            load_s(t, sA);
            float pm = -INFINITY;
            if (good) {
                if (!__all_sync(0xffffffffu, nxt_full)) apply_mask(sA, nxt_bits);
                pm = half_max(sA);
                sh->red_max[t & 1][half][il] = pm;
            }
            if (!bar_and(bar_id, 64, good)) {
                ok = false;
                break;
            }
            float m_run = fmaxf(pm, sh->red_max[t & 1][half ^ 1][il]) * sl2;  // -inf stays -inf
            float l_run = 0.0f;
            float mref = (m_run == -INFINITY) ? 0.0f : m_run;

            // One pipeline step on tile j (global tile t): load + mask + reduce tile j+1
            // while the exps of tile j run, hand P_j to the MMA, then agree on the
            // reference max of tile j+1.  Returns false when the pair must leave.
            auto step = [&](float(&cur)[64], float(&nxt)[64], int j) -> bool {
                const bool has_next = j + 1 < d.n;
                const int b = t & 1;
                bool nf = true;
                uint64_t nbits = ~0ull;
                if (has_next) {
                    load_s(t + 1, nxt);
                    make_mask(j + 1, nf, nbits);
                    if (j + 2 < d.n) fetch_meta(j + 2);
                }
                // P[b] may still be read by the PV of tile t-2
                if (good && t >= 2 &&
                    !__all_sync(0xffffffffu, mbar_wait(&sh->p_free[b], ((t - 2) >> 1) & 1, lim, abort)))
                    fail();
                float pmn = -INFINITY;
                if (good) {
                    uint32_t pk[32];
                    float ls;
                    if (!has_next) {
                        ls = exps(cur, mref, pk);
                    } else if (__all_sync(0xffffffffu, nf)) {
                        ls = exps(cur, mref, pk);
                        pmn = half_max(nxt);
                    } else {
                        apply_mask(nxt, nbits);
                        ls = exps(cur, mref, pk);
                        pmn = half_max(nxt);
                    }
                    tmem_st32(tmem + lane_off + col_p + 64 * b, pk);
                    l_run += ls;
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&sh->p_full[b]);
                }
                if (!has_next) return true;  // the epilogue reduction decides
                const int nb2 = (t + 1) & 1;
                if (good) sh->red_max[nb2][half][il] = pmn;
                if (!bar_and(bar_id, 64, good)) return false;
                const float m_new = fmaxf(m_run, fmaxf(pmn, sh->red_max[nb2][half ^ 1][il]) * sl2);
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
                    // O must include tile t, just handed over: PV_t is the (t >> 1)-th
                    // completion of p_free[b]; PV_{t-2} completed before P_t was written.
                    if (!__all_sync(0xffffffffu, mbar_wait(&sh->p_free[b], (t >> 1) & 1, lim, abort))) {
                        fail();
                    } else {
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
                        tmem_wait_st();
                    }
                }
                mref = (m_run == -INFINITY) ? 0.0f : m_run;
                return true;
            };
            int j = 0;
            bool pair_ok = true;
            while (true) {
                pair_ok = step(sA, sB, j);
                ++j;
                ++t;
                if (!pair_ok || j >= d.n) break;
                pair_ok = step(sB, sA, j);
                ++j;
                ++t;
                if (!pair_ok || j >= d.n) break;
            }
            if (!pair_ok) {  // both warps of the pair left at the same reduction
                ok = false;
                break;
            }
            // ---- epilogue: row sum of both halves, O / l, LSE ----
            if (good) sh->red_l[half][il] = l_run;
            if (!bar_and(bar_id, 64, good)) {
                ok = false;
                break;
            }
            const int t_last = t - 1;
            // O complete: PV of the item's last tile (the phase before it, two tiles
            // back, was awaited before the last P was written).  A failure here is
            // settled at the next item's reduction.
            if (!__all_sync(0xffffffffu, mbar_wait(&sh->p_free[t_last & 1], (t_last >> 1) & 1, lim, abort))) {
                fail();
                continue;
            }
            tc_fence_after();
            uint32_t ro[D / 2];
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tmem_ld32(tmem + lane_off + col_o + 32 * c, ro + 32 * c);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&sh->o_free);  // the next item's first PV may overwrite O
            const float l_tot = l_run + sh->red_l[half ^ 1][il];
            const float inv = (l_tot > 0.0f) ? 1.0f / l_tot : 0.0f;
            if (row_ok) {
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    uint32_t w[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(ro[8 * k + 2 * q]) * inv,
                                                                        __uint_as_float(ro[8 * k + 2 * q + 1]) * inv);
                        w[q] = *reinterpret_cast<const uint32_t *>(&v2);
                    }
                    orow[k] = make_uint4(w[0], w[1], w[2], w[3]);
                }
                if (half == 0)
                    p.LSE[static_cast<size_t>(d.h) * p.S + i] =
                        (l_tot > 0.0f) ? (m_run + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
            }
            ++e;
        }
        if (!ok) {
            report(p.status, SSA_ERR_TIMEOUT);
            *abort = 1;
        }
        tc_fence_before();
        mbar_arrive(&sh->softmax_done);
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

int sm_count() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
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
    SSA_CUDA_TRY(cudaMemsetAsync(p.work_counter, 0, sizeof(int), s));
    SSA_CUDA_TRY(cudaFuncSetAttribute(sparse_attn_fwd_kernel<D>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    // setmaxnreg.inc can only draw on the registers the block was launched with: refuse
    // to launch unless the compiled kernel was given exactly the planned allocation.
    cudaFuncAttributes fa;
    SSA_CUDA_TRY(cudaFuncGetAttributes(&fa, sparse_attn_fwd_kernel<D>));
    if (fa.numRegs != kLaunchRegs) {
        set_error("sparse_attn_fwd: kernel compiled with %d registers per thread, expected %d",
                  fa.numRegs, kLaunchRegs);
        return SSA_ERR_UNSUPPORTED;
    }
    const long long items = static_cast<long long>(p.H) * p.nqb;
    const unsigned grid = static_cast<unsigned>(items < sm_count() ? items : sm_count());
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
    return kCounterBytes + 2 * static_cast<size_t>(n_heads) *
                               round_up128(static_cast<size_t>(max_vert)) * d * sizeof(uint16_t);
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
    SSA_CHECK_ARG(static_cast<int64_t>(H_q) * ((S + kBM - 1) / kBM) < (1LL << 30),
                  "sparse_attn_fwd: too many query blocks");
    const size_t need = sparse_attn_fwd_ws_bytes(H_q, plan->max_vert, d);
    SSA_CHECK_ARG(ws && aligned16(ws), "sparse_attn_fwd: ws must be a 16-byte aligned buffer");
    if (ws_bytes < need) {
        set_error("sparse_attn_fwd: workspace %zu bytes < required %zu", ws_bytes, need);
        return SSA_ERR_CAPACITY;
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
    p.work_counter = static_cast<int *>(ws);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.O = static_cast<uint16_t *>(O);
    p.LSE = LSE;
    p.status = dev_status;
    p.wait_ns = wait_limit_ns();
    uint16_t *KC = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + kCounterBytes);
    uint16_t *VC = KC + static_cast<size_t>(H_q) * p.npad * d;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d == 64 ? launch<64>(Q, K, V, KC, VC, p, s) : launch<128>(Q, K, V, KC, VC, p, s);
}
