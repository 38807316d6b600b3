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
//   sparse_attn_fwd_kernel   persistent: one CTA per SM takes work items from a global
//                            counter.  An item is a PAIR of consecutive 128-row query
//                            blocks (2p, 2p+1) of one head; the CTA walks the merged
//                            key-tile sequence of the two blocks (band windows in
//                            ascending order of their first key, then stripe tiles), so a key/value
//                            tile wanted by both blocks is staged once and feeds both.
//     warp 8         lane 0: scheduler (work counter -> ring of item descriptors) and
//                    TMA producer of the K tiles of the merged sequence; each K stage
//                    carries a flag word: which slot uses it, first/last tile of a
//                    slot within the item, end of work
//     warp 10        lane 0: TMA producer of the V tiles of the same sequence, and of
//                    each slot's Q tile at the slot's first step of the item
//                    (each blocking role has a warp of its own: single-lane loops of one
//                    warp would serialise on each other's waits)
//     warps 9, 11    MMA issuers, one per slot (warp 9 allocates tensor memory).  Each
//                    128-key tile is processed as two key regions, a (keys 0-63) and b
//                    (keys 64-127), each with its own S-ready and P-ready barrier.  For
//                    merged step u and region h, slot s issues PV of region h of its tile
//                    at u-1 (P_h written over the first 32 columns of region h of S_s),
//                    then QK^T of region h of the tile at u into the same 64 columns
//                    (N = 64).  So while the softmax works on region b, the tensor core
//                    runs region a's PV and the next tile's region-a QK^T: the softmax no
//                    longer waits for the MMAs of its own tile.  Slot 1's issuer follows
//                    slot 0's (a bracket issues only once slot 0 has issued the same one;
//                    slot 0 never waits for slot 1), which staggers the two softmaxes on
//                    the MUFU without coupling them both ways (a strict alternation made
//                    each wait for the other slot's softmax).
//     warps 0-3      softmax of slot 0 (query block 2p), one thread per query row
//     warps 4-7      softmax of slot 1 (query block 2p+1)
//                    per region: tcgen05.ld S (64 columns), element mask from the plan
//                    (FULL tiles skip it), online max/sum in fp32 (log2 domain, packed
//                    f32x2 arithmetic), P as bf16 into TMEM, lazy O rescale (only when
//                    the max grows by > 2^8); epilogue O / l -> bf16 and LSE.  A slot's
//                    epilogue runs after it has handed over the P of region a of its
//                    first tile of the next item: the tensor pipe gets that P without waiting for the
//                    epilogue, and the first PV of the next item (which overwrites O_s)
//                    waits on o_empty until the epilogue has read O_s.
// Tensor memory (512 columns): S0 0..127, S1 128..255 (region a, then b), O0 256..,
// O1 256+d...
//
// Every barrier is waited on with a counter of its own completions, and every wait
// happens only after the previous completion of the same barrier was observed by the
// waiter, so a parity never aliases two phases.  Every wait is bounded: on expiry the
// kernel records SSA_ERR_TIMEOUT, stops every role, drains its own copies and MMAs,
// frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>

#include "common.cuh"
#include "trace.h"

namespace ssa {
namespace {

constexpr int kBM = SSA_BLOCK;
constexpr int kBN = SSA_BLOCK;
// Warps 0-7 softmax (one warpgroup per slot), warps 8, 10, 11 TMA producers, warp 9 MMA
// issuer.  Registers are rebalanced with setmaxnreg: the launch gives every
// thread kLaunchRegs; the TMA/MMA warpgroup drops to kCtrlRegs and the softmax
// warpgroups rise to kSoftmaxRegs, which together use exactly the launch allocation.
constexpr int kThreads = 384;
constexpr int kSlotThreads = 128;
constexpr int kSoftmaxWarps = 8;
constexpr int kWarpTma = 8, kWarpMma0 = 9, kWarpV = 10, kWarpMma1 = 11;
constexpr int kLaunchRegs = 168, kCtrlRegs = 104, kSoftmaxRegs = 200;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kCtrlRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kRing = 4;  // work-item descriptors in flight
constexpr int kMaxStages = 6;
constexpr uint32_t kTmemCols = 512;
constexpr int kBoxBytes = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr int64_t kDrainLimitNs = 1000000000LL;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale only if the max grows by > 256x
constexpr size_t kCounterBytes = 256;     // work counter at the start of the workspace
constexpr int kMaxSmem = 232448;          // 227 KB opt-in per block

// Flag word of a K stage (one merged step).  Slot s: bit s = the slot uses this key
// tile, bit 2+s = its first tile of the item, bit 4+s = its last tile of the item.
constexpr uint32_t kStepEnd = 64;
__host__ __device__ constexpr uint32_t f_in(int s) { return 1u << s; }
__host__ __device__ constexpr uint32_t f_first(int s) { return 4u << s; }
__host__ __device__ constexpr uint32_t f_last(int s) { return 16u << s; }

template <int D>
struct Cfg {
    // K and V pipeline stages (the issue order holds every V tile for one step at most).
    static constexpr int NK = (D == 128) ? 2 : 4;
    static constexpr int NV = (D == 128) ? 3 : 5;
    static constexpr int BOXES = D / 64;
    static constexpr int TILE_BYTES = BOXES * kBoxBytes;
    static constexpr int OFF_Q = 0;  // Q tile of slot 0, then slot 1
    static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + NK * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + NV * TILE_BYTES;
    static constexpr int SMEM_BYTES = OFF_BAR + 1024 + 1024;  // barrier block + alignment slack
    static constexpr uint32_t COL_O = 256;                      // O_s at COL_O + D s
    static_assert(NK <= kMaxStages && NV <= kMaxStages, "too many stages");
    static_assert(SMEM_BYTES <= kMaxSmem, "shared memory budget exceeded");
};

struct ItemDesc {
    int h, g, end;
    int qb[2];   // query block of each slot (-1: none)
    int tp0[2];  // first plan tile of the block
    int nb[2];   // band tiles
    int ns[2];   // stripe tiles
    int slo[2];  // stripe count of the previous block (columns < 128 qb)
    int sc[2];   // stripe count of the block (columns <= min(S - 1, 128 qb + 127))
    int vp;      // offset of the head's stripe columns in vert_cols
};

struct Shared {
    uint64_t item_full[kRing], item_empty[kRing];
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[kMaxStages], k_empty[kMaxStages];
    uint64_t v_full[kMaxStages], v_empty[kMaxStages];
    uint64_t s_full[2][2], p_full[2][2];  // per slot and key region (keys 0-63, 64-127 of a tile)
    uint64_t pv_a[2];                      // PV of a tile's region a complete
    uint64_t o_full[2], o_empty[2];
    uint64_t mma_drain, softmax_done;
    ItemDesc items[kRing];
    uint32_t kflags[kMaxStages];
    uint32_t tmem_base;
    int abort;
    int lead;  // brackets issued by slot 0's issuer (slot 1 follows it)
};
static_assert(sizeof(Shared) <= 1024, "barrier block too large");

struct AttnParams {
    int S, H, Hkv, nqb, npad;
    const int32_t *tile_ptr;
    const int32_t *tile_key0;
    const uint64_t *tile_dmask;
    const uint64_t *tile_cmask;
    const uint32_t *tile_flags;
    const uint64_t *tile_bits;  // Case-2 plans: element bitmaps (flag 2 tiles), else null
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
    int o_align32;  // O is 32-byte aligned (rows are then too: d * 2 bytes is a multiple of 32)
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
// Attention forward (persistent, two query blocks per work item)
// ---------------------------------------------------------------------------------

// Work item idx -> descriptor of the pair of query blocks (2 pq, 2 pq + 1) of head h.
// Items come in groups of G = H / H_kv consecutive heads (the heads that share one KV
// head under the default map); within a group the pairs run from the last down (later
// blocks hold more tiles under causal patterns) with the group's heads side by side.
// The CTAs then work on one KV head at a time, so the band windows that consecutive
// pairs of a head share are still in L2 when the later pair reads them.
__device__ ItemDesc make_pair(const AttnParams &p, int idx) {
    ItemDesc d;
    const int npair = (p.nqb + 1) >> 1;
    const int G = max(1, p.H / p.Hkv);
    const int grp = idx / (npair * G);
    const int h0 = grp * G;
    const int gsz = min(G, p.H - h0);  // the last group may be short
    const int rem = idx - grp * npair * G;
    const int pq = npair - 1 - rem / gsz;
    d.h = h0 + rem % gsz;
    d.g = kv_head(p, d.h);
    d.end = 0;
    const bool bad = d.g < 0 || d.g >= p.Hkv;
    if (bad) report(p.status, SSA_ERR_INVALID);  // its rows still get O = 0, LSE = -inf
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const int qb = 2 * pq + s;
        d.qb[s] = -1;
        d.tp0[s] = d.nb[s] = d.ns[s] = d.slo[s] = d.sc[s] = 0;
        if (qb >= p.nqb) continue;
        d.qb[s] = qb;
        const int it = d.h * p.nqb + qb;
        d.tp0[s] = __ldg(p.tile_ptr + it);
        d.slo[s] = qb > 0 ? __ldg(p.stripe_cnt + it - 1) : 0;
        d.sc[s] = __ldg(p.stripe_cnt + it);
        if (!bad) {
            d.nb[s] = __ldg(p.tile_ptr + it + 1) - d.tp0[s];
            d.ns[s] = (d.sc[s] + kBN - 1) / kBN;
        }
    }
    d.vp = __ldg(p.vert_ptr + d.h);
    return d;
}

// The merged key-tile sequence of an item: band tiles of both blocks in ascending order
// of their first key (a window listed by both, same start, is one step), then the
// stripe tiles (block 2p+1 holds at least as many stripe columns as block 2p).  The next band entry of each block is
// loaded one step ahead so the producers do not wait on it.
struct Steps {
    const int32_t *key0[2];  // window start keys of each block's band tiles
    int nb[2], ns[2], i[2], a[2], an[2];
    int js;
    bool started[2], emitted;
};

__device__ __forceinline__ void steps_init(Steps &st, const AttnParams &p, const ItemDesc &d) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        st.key0[s] = p.tile_key0 + d.tp0[s];
        st.nb[s] = d.nb[s];
        st.ns[s] = d.ns[s];
        st.i[s] = 0;
        st.a[s] = d.nb[s] > 0 ? __ldg(st.key0[s]) : INT_MAX;
        st.an[s] = d.nb[s] > 1 ? __ldg(st.key0[s] + 1) : INT_MAX;
        st.started[s] = false;
    }
    st.js = 0;
    st.emitted = false;
}

// Next step of the sequence: key-tile row, whether it is a band tile (else a stripe
// tile of K_C / V_C) and the slot flags.  Returns false after the last step.  An item
// without any tile yields one no-op step (row0 < 0, no slot, no data): the MMA issuer
// then still passes a step boundary between the items around it, where it issues the
// PVs the previous item's epilogue waits for.
__device__ __forceinline__ bool steps_next(Steps &st, bool &band, int &row0, uint32_t &flags) {
    flags = 0;
    const bool first = !st.emitted;
    st.emitted = true;
    if (st.a[0] != INT_MAX || st.a[1] != INT_MAX) {
        const int key0 = min(st.a[0], st.a[1]);
        band = true;
        row0 = key0;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            if (st.a[s] != key0) continue;
            flags |= f_in(s);
            if (!st.started[s]) {
                flags |= f_first(s);
                st.started[s] = true;
            }
            ++st.i[s];
            st.a[s] = st.an[s];
            st.an[s] = (st.i[s] + 1 < st.nb[s]) ? __ldg(st.key0[s] + st.i[s] + 1) : INT_MAX;
            if (st.i[s] == st.nb[s] && st.ns[s] == 0) flags |= f_last(s);
        }
        return true;
    }
    if (st.js < max(st.ns[0], st.ns[1])) {
        band = false;
        row0 = st.js * kBN;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            if (st.js >= st.ns[s]) continue;
            flags |= f_in(s);
            if (!st.started[s]) {
                flags |= f_first(s);
                st.started[s] = true;
            }
            if (st.js == st.ns[s] - 1) flags |= f_last(s);
        }
        ++st.js;
        return true;
    }
    if (first) {  // no tile at all
        band = false;
        row0 = -1;
        return true;
    }
    return false;
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
    const int n_items = p.H * ((p.nqb + 1) >> 1);

    if (threadIdx.x == 0) {
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&sh->item_full[r], 1);
            mbar_init(&sh->item_empty[r], 1 + kSoftmaxWarps);  // Q/V producer, softmax warps
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh->q_full[s], 1);
            mbar_init(&sh->q_empty[s], 1);
            for (int h = 0; h < 2; ++h) {
                mbar_init(&sh->s_full[s][h], 1);
                mbar_init(&sh->p_full[s][h], kSlotThreads);
            }
            mbar_init(&sh->pv_a[s], 1);
            mbar_init(&sh->o_full[s], 1);
            mbar_init(&sh->o_empty[s], kSlotThreads);
        }
        for (int st = 0; st < C::NK; ++st) {
            mbar_init(&sh->k_full[st], 1);
            mbar_init(&sh->k_empty[st], 2);  // one arrival per slot's MMA issuer
        }
        for (int st = 0; st < C::NV; ++st) {
            mbar_init(&sh->v_full[st], 1);
            mbar_init(&sh->v_empty[st], 2);
        }
        mbar_init(&sh->mma_drain, 2);
        mbar_init(&sh->softmax_done, 2 * kSlotThreads);
        sh->abort = 0;
        sh->lead = 0;
        fence_barrier_init();
    }
    if (warp == kWarpMma0) {
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
            // ----------------- scheduler + K producer (warp 8, lane 0) -----------------
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmKC);
            bool ok = true;
            int m = 0, tk = 0;
            while (ok) {
                // take the next work item and publish its descriptor to the other roles
                const int idx = atomicAdd(p.work_counter, 1);
                const int slot = m % kRing;
                if (m >= kRing && !mbar_wait(&sh->item_empty[slot], ((m / kRing) - 1) & 1, lim, abort)) {
                    ok = false;
                    break;
                }
                ItemDesc d;
                if (idx < n_items) {
                    d = make_pair(p, idx);
                } else {
                    d.end = 1;
                }
                sh->items[slot] = d;
                mbar_arrive(&sh->item_full[slot]);  // release: the descriptor is visible
                ++m;
                if (d.end) break;
                Steps st;
                steps_init(st, p, d);
                bool band;
                int row0;
                uint32_t fl;
                while (steps_next(st, band, row0, fl)) {
                    const int si = tk % C::NK;
                    if (tk >= C::NK && !mbar_wait(&sh->k_empty[si], ((tk / C::NK) - 1) & 1, lim, abort)) {
                        ok = false;
                        break;
                    }
                    sh->kflags[si] = fl;
                    if (row0 < 0) {  // no-op step: no data
                        mbar_arrive(&sh->k_full[si]);
                    } else {
                        uint8_t *dst = smem + C::OFF_K + si * C::TILE_BYTES;
                        mbar_arrive_expect_tx(&sh->k_full[si], C::TILE_BYTES);
                        for (int b = 0; b < C::BOXES; ++b)
                            tma_load_3d(dst + b * kBoxBytes, band ? &tmK : &tmKC, &sh->k_full[si], 64 * b, row0,
                                        band ? d.g : d.h);
                    }
                    ++tk;
                }
            }
            if (ok) {  // end-of-work step for the MMA issuer (no data)
                const int si = tk % C::NK;
                if (tk >= C::NK && !mbar_wait(&sh->k_empty[si], ((tk / C::NK) - 1) & 1, lim, abort)) {
                    ok = false;
                } else {
                    sh->kflags[si] = kStepEnd;
                    mbar_arrive(&sh->k_full[si]);
                    ++tk;
                }
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            // Drain: never leave the CTA with a copy still writing shared memory.
            for (int u = (tk > C::NK ? tk - C::NK : 0); u < tk; ++u)
                mbar_wait(&sh->k_full[u % C::NK], (u / C::NK) & 1, kDrainLimitNs, nullptr);
        }
      } else if (warp == kWarpV) {
        if (lane == 0) {
            // ------------------------- Q and V producer -------------------------
            // The V tiles of the merged sequence, and each slot's Q tile at the slot's
            // first step of the item.  A Q tile waits for the last QK^T of its slot in
            // the previous item; loading it only at the slot's first step keeps the V
            // tiles of the steps before it from waiting on that QK^T.
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmVC);
            bool ok = true;
            int m = 0, tv = 0;
            int qn[2] = {0, 0};
            while (ok) {
                const int slot = m % kRing;
                if (!mbar_wait(&sh->item_full[slot], (m / kRing) & 1, lim, abort)) {
                    ok = false;
                    break;
                }
                const ItemDesc d = sh->items[slot];
                mbar_arrive(&sh->item_empty[slot]);
                ++m;
                if (d.end) break;
                Steps st;
                steps_init(st, p, d);
                bool band;
                int row0;
                uint32_t fl;
                while (steps_next(st, band, row0, fl)) {
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        if (!ok || !(fl & f_first(s))) continue;
                        if (qn[s] >= 1 && !mbar_wait(&sh->q_empty[s], (qn[s] - 1) & 1, lim, abort)) {
                            ok = false;
                            continue;
                        }
                        uint8_t *sQ = smem + C::OFF_Q + s * C::TILE_BYTES;
                        mbar_arrive_expect_tx(&sh->q_full[s], C::TILE_BYTES);
                        for (int b = 0; b < C::BOXES; ++b)
                            tma_load_3d(sQ + b * kBoxBytes, &tmQ, &sh->q_full[s], 64 * b, d.qb[s] * kBM, d.h);
                        ++qn[s];
                    }
                    if (!ok) break;
                    const int si = tv % C::NV;
                    if (tv >= C::NV && !mbar_wait(&sh->v_empty[si], ((tv / C::NV) - 1) & 1, lim, abort)) {
                        ok = false;
                        break;
                    }
                    if (row0 < 0) {  // no-op step: no data
                        mbar_arrive(&sh->v_full[si]);
                    } else {
                        uint8_t *dst = smem + C::OFF_V + si * C::TILE_BYTES;
                        mbar_arrive_expect_tx(&sh->v_full[si], C::TILE_BYTES);
                        for (int b = 0; b < C::BOXES; ++b)
                            tma_load_3d(dst + b * kBoxBytes, band ? &tmV : &tmVC, &sh->v_full[si], 64 * b, row0,
                                        band ? d.g : d.h);
                    }
                    ++tv;
                }
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            // Drain: never leave the CTA with a copy still writing shared memory.
            for (int u = (tv > C::NV ? tv - C::NV : 0); u < tv; ++u)
                mbar_wait(&sh->v_full[u % C::NV], (u / C::NV) & 1, kDrainLimitNs, nullptr);
            for (int s = 0; s < 2; ++s)
                if (qn[s] >= 1) mbar_wait(&sh->q_full[s], (qn[s] - 1) & 1, kDrainLimitNs, nullptr);
        }
      } else if (warp == kWarpMma0 || warp == kWarpMma1) {
        // ------------------------------ MMA issuers ------------------------------
        // One thread per slot (warps 9 and 11, on different SM sub-partitions), each
        // issuing only its own slot's tcgen05.mma.  A tcgen05.mma blocks its thread while
        // the tensor pipe's short queue is full, so a single issuer leaves the pipe idle
        // whenever it does its waits and commits; with two, one slot's MMAs run while
        // the other's issuer does its bookkeeping.  Per merged step u, slot s, region h:
        //   PV_h of its tile at u-1 (if any) | (region a: wait K_u) | QK_h(u) (if s uses K_u)
        // A region's QK^T always follows the PV of the same region of the previous tile
        // (P_h shares the region's columns; tcgen05.mma of one thread execute in issue
        // order).  After the PV of region a the issuer commits pv_a, which the softmax
        // waits for only when it has to rescale O at region b.  Every PV is issued
        // at the step after its QK^T, so no V tile is held longer than one step.  Each
        // issuer releases every K and V stage once (a commit after its own MMAs on it,
        // else a plain arrival), so each stage's empty barrier takes two arrivals; the
        // K ring bounds the distance between the two issuers to NK steps, and NV > NK
        // keeps every arrival in the phase it belongs to.  Every release of a stage
        // (commit or plain arrival) comes after the issuer observed that stage's fill for
        // the step, so no release can complete the stage's previous phase early, and a
        // producer never waits more than one phase behind.
        if (lane == 0) {
            const int s = (warp == kWarpMma1) ? 1 : 0;
            constexpr uint32_t IDESC_QK = idesc_bf16(kBM, kBN / 2, false);  // one key region: N = 64
            constexpr uint32_t IDESC_PV = idesc_bf16(kBM, D, true);
            const uint32_t sQ = smem_u32(smem + C::OFF_Q + s * C::TILE_BYTES);
            const uint32_t tS = tmem + 128 * s, tO = tmem + C::COL_O + D * s;
            bool ok = true;
            int u = 0;  // merged step (K and V ring index)
            int qcnt = 0, pcnt = 0, ocnt = 0;  // ocnt: first PVs of items issued
            bool pend = false, pfirst = false, plast = false;
            // The issuer polls (mbar_wait_poll): mbarrier.try_wait in a thread with MMAs
            // in flight costs about their drain time even when the phase is complete.
            auto wait = [&](uint64_t *bar, int parity) {
                if (ok && !mbar_wait_poll(bar, parity, lim, abort)) ok = false;
                return ok;
            };
            while (ok) {
                const int v = u - 1;
                uint32_t f = 0;
                bool end = false, in = false;
                // Two brackets per merged step, one per key region h (keys 64 h .. 64 h + 63):
                // PV of region h of the slot's tile at u-1 (reads P_h, written over the first
                // 32 columns of region h of S_s), then QK^T of region h of the tile at u into
                // the same region.  Region a's MMAs run while the softmax works on region b.
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    // 1. every wait of this bracket, while the other slot's MMAs run
                    if (h == 0 && u >= 1 && !wait(&sh->v_full[v % C::NV], (v / C::NV) & 1)) break;
                    if (pend && !wait(&sh->p_full[s][h], pcnt & 1)) break;
                    // the first PV of an item overwrites O_s: the previous item's epilogue
                    // must have read it
                    if (h == 0 && pend && pfirst && ocnt >= 1 && !wait(&sh->o_empty[s], (ocnt - 1) & 1)) break;
                    if (h == 0) {
                        if (!wait(&sh->k_full[u % C::NK], (u / C::NK) & 1)) break;
                        f = sh->kflags[u % C::NK];
                        end = (f & kStepEnd) != 0;
                        in = !end && (f & f_in(s));
                        if (in && (f & f_first(s)) && !wait(&sh->q_full[s], qcnt & 1)) break;
                    }
                    // slot 1 follows slot 0: a bracket issues only after slot 0 issued it
                    if (s == 1 && ok) {
                        volatile int *lead = &sh->lead;
                        const int want = 2 * u + h + 1;
                        if (*lead < want) {
                            const uint64_t t0 = global_timer_ns();
                            while (*lead < want) {
                                if (*abort || static_cast<int64_t>(global_timer_ns() - t0) >= lim) {
                                    ok = false;
                                    break;
                                }
                            }
                        }
                        if (!ok) break;
                    }
                    // 2. PV of region h of the slot's tile at u-1, then QK^T of region h of the
                    // tile at u
                    tc_fence_after();
                    if (pend) {
                        const uint32_t sV = smem_u32(smem + C::OFF_V + (v % C::NV) * C::TILE_BYTES);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            // B = V tile, MN-major: 16 keys per step (2 x 8-row groups of 128 B)
                            const int kk = 4 * h + q;
                            umma_ts(tO, tS + 64 * h + 8 * q, sdesc(sV + kk * 2048, kBoxBytes, 1024), IDESC_PV,
                                    (!pfirst || kk > 0) ? 1u : 0u);
                        }
                        if (h == 0) umma_commit(&sh->pv_a[s]);
                    }
                    if (in) {
                        // key rows 64 h .. 64 h + 63 of the K tile start 8 KB into each box
                        const uint32_t sK = smem_u32(smem + C::OFF_K + (u % C::NK) * C::TILE_BYTES) + 8192 * h;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            // A = Q, B = K rows, both K-major: 16 elements = 32 B per step
                            const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
                            umma_ss(tS + 64 * h, sdesc(sQ + off, 16, 1024), sdesc(sK + off, 16, 1024), IDESC_QK,
                                    kk > 0 ? 1u : 0u);
                        }
                    }
                    // 3. completions.  A release of V_(u-1) by a slot that did not read it comes
                    // after its fill was observed above: the fill of step u-1 follows the
                    // completion of the stage's previous phase, so the release lands in the
                    // phase of step u-1 (never in the previous one, where it would stand in
                    // for the other slot's PV still reading the stage, and never a phase
                    // ahead of the producer, as for a no-op step that no slot reads).
                    if (s == 0) *reinterpret_cast<volatile int *>(&sh->lead) = 2 * u + h + 1;
                    if (in) umma_commit(&sh->s_full[s][h]);
                    if (h == 1) {
                        if (pend) {
                            if (plast) umma_commit(&sh->o_full[s]);  // O_s of the item complete
                            umma_commit(&sh->v_empty[v % C::NV]);    // completes once the PVs have read V
                            if (pfirst) ++ocnt;
                            ++pcnt;
                        } else if (u >= 1) {
                            mbar_arrive(&sh->v_empty[v % C::NV]);
                        }
                        if (in) {
                            if (f & f_last(s)) umma_commit(&sh->q_empty[s]);  // Q_s no longer read
                            umma_commit(&sh->k_empty[u % C::NK]);
                            if (f & f_first(s)) ++qcnt;
                        } else if (!end) {
                            mbar_arrive(&sh->k_empty[u % C::NK]);
                        }
                    }
                }
                if (!ok || end) break;
                pend = in;
                if (in) {
                    pfirst = (f & f_first(s)) != 0;
                    plast = (f & f_last(s)) != 0;
                }
                ++u;
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            umma_commit(&sh->mma_drain);  // completes once every MMA this thread issued is done
        }
        __syncwarp();
        // Free tensor memory after the softmax warps are done and every MMA has finished.
        if (warp == kWarpMma0) {
            if (lane == 0) {
                mbar_wait(&sh->softmax_done, 0, kDrainLimitNs, nullptr);
                mbar_wait(&sh->mma_drain, 0, kDrainLimitNs, nullptr);
            }
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, kTmemCols);
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // -------------------------------- softmax / epilogue -------------------------------
        // Warpgroup s owns slot s: thread il of the warpgroup owns query row 128 qb + il
        // and TMEM lane il (warp w may only touch lanes 32 (w % 4) ..).
        const int s = warp >> 2;
        const int quarter = warp & 3;
        const int il = 32 * quarter + lane;
        const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
        const uint32_t tS = tmem + lane_off + 128u * s;           // S_s; P_s in its first 64 columns
        const uint32_t tO = tmem + lane_off + C::COL_O + D * s;   // O_s
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        constexpr uint32_t kNegInf = 0xff800000u;
        bool ok = true;
        int m = 0, tcnt = 0, icnt = 0;
        // The epilogue of the slot's last item with tiles, owed until the P of the first
        // tile of the slot's next such item (or the end of work): row e_i of head e_h,
        // with its running max and sum.
        bool owed = false;
        int e_h = 0, e_i = 0;
        float e_m = 0.0f, e_l = 0.0f;
        auto epilogue = [&]() -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(&sh->o_full[s], icnt & 1, lim, abort))) return false;
            ++icnt;
            tc_fence_after();
            uint32_t ro[D];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + 32 * c, ro + 32 * c);
            tmem_wait_ld();
            // O_s is read: the next item's first PV may overwrite it
            tc_fence_before();
            mbar_arrive(&sh->o_empty[s]);
            // a row whose max stayed -inf has no retained key: O = 0, LSE = -inf
            const bool empty = !(e_m > -INFINITY) || !(e_l > 0.0f);
            const float inv = empty ? 0.0f : 1.0f / e_l;
            if (e_i < p.S) {
                const size_t row = static_cast<size_t>(e_h) * p.S + e_i;
                uint4 *orow = reinterpret_cast<uint4 *>(p.O + row * D);
                // the row as bf16, 16 columns (32 bytes) per store when O allows it: half the
                // store instructions of 16-byte stores for the same bytes
                uint32_t w[D / 2];
#pragma unroll
                for (int q = 0; q < D / 2; ++q) {
                    const __nv_bfloat162 v2 =
                        __floats2bfloat162_rn(__uint_as_float(ro[2 * q]) * inv, __uint_as_float(ro[2 * q + 1]) * inv);
                    w[q] = *reinterpret_cast<const uint32_t *>(&v2);
                }
                if (p.o_align32) {
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) st_global_v8(orow + 2 * k, w + 8 * k);
                } else {
#pragma unroll
                    for (int k = 0; k < D / 8; ++k) orow[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                }
                p.LSE[row] =
                    empty ? -INFINITY : (e_m + log2f(e_l)) * 0.69314718055994531f;
            }
            return true;
        };
        while (true) {
            const int slot = m % kRing;
            if (!__all_sync(0xffffffffu, mbar_wait(&sh->item_full[slot], (m / kRing) & 1, lim, abort))) {
                ok = false;
                break;
            }
            const ItemDesc d = sh->items[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->item_empty[slot]);
            ++m;
            if (d.end) break;
            const int qb = s ? d.qb[1] : d.qb[0];
            if (qb < 0) continue;
            const int nb = s ? d.nb[1] : d.nb[0];
            const int ns = s ? d.ns[1] : d.ns[0];
            const int tp0 = s ? d.tp0[1] : d.tp0[0];
            const int slo = s ? d.slo[1] : d.slo[0];
            const int n = nb + ns;
            const int i = qb * kBM + il;
            const bool row_ok = i < p.S;
            if (n == 0) {  // no retained key in this block: O = 0, LSE = -inf
                if (row_ok) {
                    uint4 *orow = reinterpret_cast<uint4 *>(p.O + (static_cast<size_t>(d.h) * p.S + i) * D);
#pragma unroll
                    for (int k = 0; k < D / 8; ++k) orow[k] = make_uint4(0, 0, 0, 0);
                    p.LSE[static_cast<size_t>(d.h) * p.S + i] = -INFINITY;
                }
                continue;
            }
            // stripe columns c <= i: between the counts of the previous and this block
            // (usually none or a few: a short count, else a binary search)
            int n_i = 0;
            if (row_ok && ns > 0) {
                const int32_t *Ch = p.vert_cols + d.vp + slo;
                const int nc = (s ? d.sc[1] : d.sc[0]) - slo;
                if (nc <= 8) {
                    n_i = slo;
                    for (int t = 0; t < nc; ++t) n_i += (__ldg(Ch + t) <= i) ? 1 : 0;
                } else {
                    n_i = slo + lower_bound_i32(Ch, nc, i + 1);
                }
            }
            // plan data of band tile j: pulled into L1 one tile ahead, loaded at the tile
            auto prefetch_l1 = [&](int j) {
                if (j < nb) {
                    const size_t tt = static_cast<size_t>(tp0 + j);
                    asm volatile("prefetch.global.L1 [%0];" ::"l"(p.tile_dmask + 4 * tt));
                    asm volatile("prefetch.global.L1 [%0];" ::"l"(p.tile_cmask + 2 * tt));
                    asm volatile("prefetch.global.L1 [%0];" ::"l"(p.tile_flags + tt));
                }
            };
            uint32_t mf = 0;
            uint64_t md[4] = {0, 0, 0, 0}, mc[2] = {0, 0};
            auto fetch = [&](int j) {
                if (j < nb) {
                    const size_t tt = static_cast<size_t>(tp0 + j);
                    mf = __ldg(p.tile_flags + tt);
                    const ulonglong2 d01 = __ldg(reinterpret_cast<const ulonglong2 *>(p.tile_dmask + 4 * tt));
                    const ulonglong2 d23 = __ldg(reinterpret_cast<const ulonglong2 *>(p.tile_dmask + 4 * tt) + 1);
                    const ulonglong2 c01 = __ldg(reinterpret_cast<const ulonglong2 *>(p.tile_cmask + 2 * tt));
                    md[0] = d01.x;
                    md[1] = d01.y;
                    md[2] = d23.x;
                    md[3] = d23.y;
                    mc[0] = c01.x;
                    mc[1] = c01.y;
                }
            };
            prefetch_l1(0);
            float m_run = -INFINITY, l_run = 0.0f;
            for (int j = 0; j < n; ++j) {
                // this tile's row mask (bit k = key column k), then prefetch the next tile's
                bool full;
                uint64_t mlo, mhi;
                fetch(j);
                if (j < nb) {
                    full = (mf & 1u) != 0;
                    if (mf & 2u) {
                        // element-bitmap tile (Case 2): the row's 128 bits, slot in dmask word 0
                        const ulonglong2 b =
                            __ldg(reinterpret_cast<const ulonglong2 *>(p.tile_bits) + md[0] * kBM + il);
                        mlo = b.x;
                        mhi = b.y;
                    } else {
                        row_diag_mask(md, il, mlo, mhi);
                        mlo &= ~mc[0];
                        mhi &= ~mc[1];
                    }
                    if (!row_ok) mlo = mhi = 0;
                } else {
                    const int lk = n_i - (j - nb) * kBN;  // key column k active iff k < lk
                    full = lk >= kBN;
                    mlo = lk >= 64 ? ~0ull : (lk <= 0 ? 0ull : (1ull << lk) - 1ull);
                    mhi = lk >= 128 ? ~0ull : (lk <= 64 ? 0ull : (1ull << (lk - 64)) - 1ull);
                }
                prefetch_l1(j + 1);
                // the tile's two key regions in order; each is a step of the online softmax
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&sh->s_full[s][h], tcnt & 1, lim, abort))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t mk = h ? mhi : mlo;
                    const bool do_mask = !__all_sync(0xffffffffu, full || mk == ~0ull);
                    uint32_t r[64];
                    tmem_ld32(tS + 64 * h, r);
                    tmem_ld32(tS + 64 * h + 32, r + 32);
                    tmem_wait_ld();
                    if (do_mask) {
                        const uint32_t w0 = static_cast<uint32_t>(mk), w1 = static_cast<uint32_t>(mk >> 32);
#pragma unroll
                        for (int k = 0; k < 64; ++k)
                            r[k] = (((k < 32 ? w0 : w1) >> (k & 31)) & 1u) ? r[k] : kNegInf;
                    }
                    float a[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) a[q] = fmaxf(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
#pragma unroll
                    for (int k = 16; k < 64; k += 16) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            a[q] = fmax3(a[q], __uint_as_float(r[k + 2 * q]), __uint_as_float(r[k + 2 * q + 1]));
                    }
                    const float tmax = fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
                    // lazy rescale rule: a new reference only when the row max grows by more
                    // than 2^8
                    const float m_new = fmaxf(m_run, tmax * sl2);  // -inf stays -inf
                    const bool grow = (m_new != -INFINITY) && (m_run == -INFINITY || m_new > m_run + kRescaleThreshold);
                    const bool need_o = grow && (m_run != -INFINITY);
                    float factor = 1.0f;
                    if (grow) {
                        factor = (m_run == -INFINITY) ? 0.0f : ex2_approx(m_run - m_new);
                        l_run *= factor;
                        m_run = m_new;
                    }
                    // P = 2^(s * scale_log2 - mref) over the region as packed bf16 pairs, over
                    // the region's first 32 columns
                    {
                        const float mref = (m_run == -INFINITY) ? 0.0f : m_run;
                        const uint64_t nm2 = f2_pack(-mref, -mref);
                        uint64_t acc[4] = {0, 0, 0, 0};
                        uint32_t pk[32];
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), sl2x2, nm2),
                                      x0, x1);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            acc[k & 3] = f2_add(acc[k & 3], f2_pack(p0, p1));
                            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                            pk[k] = *reinterpret_cast<const uint32_t *>(&pb);
                        }
                        tmem_st32(tS + 64 * h, pk);
                        float a0, a1, a2, a3, a4, a5, a6, a7;
                        f2_unpack(acc[0], a0, a1);
                        f2_unpack(acc[1], a2, a3);
                        f2_unpack(acc[2], a4, a5);
                        f2_unpack(acc[3], a6, a7);
                        l_run += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
                    }
                    if (__any_sync(0xffffffffu, need_o)) {
                        // O_s must hold every PV taken against the old reference, and none
                        // against the new one.  Region a: the PV of region b of the previous
                        // tile precedes this tile's region-b QK^T (s_full[s][1]).  Region b:
                        // the PV of this tile's region a (pv_a), whose P the warps have handed
                        // over.  This tile's P of region h is not handed over yet.
                        const bool okw = h == 0 ? mbar_wait(&sh->s_full[s][1], tcnt & 1, lim, abort)
                                                : mbar_wait(&sh->pv_a[s], tcnt & 1, lim, abort);
                        if (!__all_sync(0xffffffffu, okw)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const float f = need_o ? factor : 1.0f;
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tO + 32 * c, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
                            tmem_st32(tO + 32 * c, o);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&sh->p_full[s][h]);
                    // the previous item's epilogue, now that the tensor pipe has the P of
                    // this item's first region (its first PV waits for O_s to be read)
                    if (j == 0 && h == 0 && owed) {
                        if (!epilogue()) {
                            ok = false;
                            break;
                        }
                        owed = false;
                    }
                }
                if (!ok) break;
                ++tcnt;
            }
            if (!ok) break;
            owed = true;
            e_h = d.h;
            e_i = i;
            e_m = m_run;
            e_l = l_run;
        }
        if (ok && owed && !epilogue()) ok = false;
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
    // Once per device: the shared-memory opt-in, and a check that the compiled kernel was
    // given exactly the planned register allocation (setmaxnreg.inc can only draw on the
    // registers the block was launched with).
    static std::atomic<uint64_t> ready{0};
    int dev = 0;
    SSA_CUDA_TRY(cudaGetDevice(&dev));
    const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0;
    if (!bit || !(ready.load() & bit)) {
        SSA_CUDA_TRY(cudaFuncSetAttribute(sparse_attn_fwd_kernel<D>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
        cudaFuncAttributes fa;
        SSA_CUDA_TRY(cudaFuncGetAttributes(&fa, sparse_attn_fwd_kernel<D>));
        if (fa.numRegs != kLaunchRegs) {
            set_error("sparse_attn_fwd: kernel compiled with %d registers per thread, expected %d",
                      fa.numRegs, kLaunchRegs);
            return SSA_ERR_UNSUPPORTED;
        }
        ready.fetch_or(bit);
    }
    const long long items = static_cast<long long>(p.H) * ((p.nqb + 1) / 2);
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
    ssa::TraceRange trace_range("sparse_attn_fwd");
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
    SSA_CHECK_ARG(plan->tile_ptr && plan->tile_key0 && plan->tile_dmask && plan->tile_cmask &&
                      plan->tile_flags && plan->stripe_cnt && plan->ext_vert_ptr &&
                      plan->ext_vert_cols,
                  "sparse_attn_fwd: null plan array");
    SSA_CHECK_ARG(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O),
                  "sparse_attn_fwd: Q, K, V and O must be 16-byte aligned");
    SSA_CHECK_ARG(aligned16(plan->tile_dmask) && aligned16(plan->tile_cmask),
                  "sparse_attn_fwd: plan tile_dmask and tile_cmask must be 16-byte aligned");
    SSA_CHECK_ARG(plan->bitmap_slots == 0 || (plan->tile_bits && aligned16(plan->tile_bits)),
                  "sparse_attn_fwd: a Case-2 plan needs tile_bits (16-byte aligned)");
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
    p.tile_key0 = plan->tile_key0;
    p.tile_dmask = plan->tile_dmask;
    p.tile_cmask = plan->tile_cmask;
    p.tile_flags = plan->tile_flags;
    p.tile_bits = plan->tile_bits;
    p.stripe_cnt = plan->stripe_cnt;
    p.vert_ptr = plan->ext_vert_ptr;
    p.vert_cols = plan->ext_vert_cols;
    p.kv_map = kv_map;
    p.work_counter = static_cast<int *>(ws);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.O = static_cast<uint16_t *>(O);
    p.o_align32 = (reinterpret_cast<uintptr_t>(O) & 31u) == 0;
    p.LSE = LSE;
    p.status = dev_status;
    p.wait_ns = wait_limit_ns();
    uint16_t *KC = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + kCounterBytes);
    uint16_t *VC = KC + static_cast<size_t>(H_q) * p.npad * d;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return d == 64 ? launch<64>(Q, K, V, KC, VC, p, s) : launch<128>(Q, K, V, KC, VC, p, s);
}
