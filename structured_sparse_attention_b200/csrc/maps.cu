// maps.cu -- stage one, step 1: averaged causal attention maps at capture length L.
//
// Stage one of DAM starts from attention maps averaged over a calibration corpus at
// L = 512 (DAM review page: "What carries the argument"; "Assumptions & free
// parameters").  This kernel produces them on the GPU from B samples of per-head Q, K:
//   maps[m][i][j] = (1/B) sum_b softmax_j(scale * Q[m][b][i] . K[m][b][j])   (j <= i)
//   maps[m][i][j] = 0                                                        (j > i)
// in the layout sparse_pattern_capture reads.
//
// Work items are (map, 128-row block rb), run by persistent CTAs (one per SM) whose
// pipelines carry on from item to item; the row block's keys are the chunks c = 0..rb of
// 128 keys, and a tile is one 128 x 128 block S = Q_b K_(b,c)^T (tcgen05, fp32 in TMEM):
//   pass 1 (samples outer, chunks inner): per row the running max and sum of 2^(x - max)
//          over the causal keys of sample b  ->  (m_b, 1 / l_b) kept in shared memory
//   pass 2 (chunks outer, samples inner): the same tiles again; P = 2^(x - m_b) / l_b
//          accumulated in registers over the samples, then the chunk of the map row is
//          written once.
// Each exponential is taken twice (once per pass): accumulating a whole row block over
// all its chunks at once would need (rb + 1) x 128 fp32 values per row.
//
// Roles (576 threads): warps 0-15 softmax, four warpgroups splitting each tile's columns
// (part h takes columns 32h..32h+31; thread il of a warpgroup owns row 128 rb + il,
// TMEM lane il), so four warps per SM sub-partition share the MUFU and hide each
// other's latencies; the parts' running max and sum are combined through shared memory
// at the end of each sample, and part 0 keeps (m_b, 1 / l_b); at d = 64 each part sends
// its 32 columns of a finished chunk to the map with a TMA store from a swizzled staging
// buffer.  Warp 16 lane 0: TMA producer of the Q block and K chunk of each tile.
// Warp 17: tensor memory (four S buffers of 128 columns, so the MMAs run up to three
// tiles ahead of the softmax) and lane 0 issues the MMAs.
//
// Every wait is bounded: on expiry the kernel records SSA_ERR_TIMEOUT, stops every role,
// drains its copies and MMAs, frees tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "trace.h"

namespace ssa {
namespace {

constexpr int kMapsMaxB = SSA_MAPS_MAX_B;
// The softmax splits every 128-column tile into kMParts column parts, one warpgroup
// each, so that kMParts warps per SM sub-partition keep the MUFU fed.
constexpr int kMParts = 4;
constexpr int kMCols = 128 / kMParts;  // columns per thread and tile
constexpr int kMSoftmaxThreads = 128 * kMParts;
constexpr int kMThreads = kMSoftmaxThreads + 64;
constexpr int kMWarpTma = kMParts * 4, kMWarpMma = kMParts * 4 + 1;
constexpr int kMSBuf = 4;  // S buffers in tensor memory: the MMA runs up to three tiles ahead
constexpr uint32_t kMTmemCols = 128 * kMSBuf;
constexpr int kMBoxBytes = 128 * 128;  // 128 rows x 64 bf16, one 128-byte swizzle span
constexpr int64_t kMDrainNs = 1000000000LL;

template <int D>
struct MCfg {
    static constexpr int NS = (D == 64) ? 3 : 2;        // smem stages (Q block + K chunk)
    // d = 64 writes the map through shared memory with TMA stores (one 32-column x
    // 128-row box per part); d = 128 has no room for the staging and stores directly
    static constexpr bool STAGED = D == 64;
    static constexpr int BOXES = D / 64;
    static constexpr int TILE = BOXES * kMBoxBytes;     // one 128-row bf16 operand
    static constexpr int STAGE = 2 * TILE;
    static constexpr int OFF_STAT = NS * STAGE;         // float2 [MAXB][128]: (m_b, 1 / l_b)
    static constexpr int OFF_XCH = OFF_STAT + kMapsMaxB * 128 * 8;  // float2 [2][kMParts][128]
    static constexpr int OFF_STG = OFF_XCH + 2 * kMParts * 128 * 8;  // [kMParts][128 rows][128 B]
    static constexpr int OFF_BAR = OFF_STG + (STAGED ? kMParts * 128 * 128 : 0);
    static constexpr int SMEM = OFF_BAR + 1024 + 1024;  // barrier block + alignment slack
    static_assert(SMEM <= 232448, "shared memory budget exceeded");
};

struct MShared {
    uint64_t full[4], empty[4];
    uint64_t s_full[kMSBuf], s_empty[kMSBuf];
    uint64_t stg_full[kMParts], stg_free[kMParts];  // staging buffer of each part
    uint64_t xch[2];
    uint64_t stat_ready;  // part 0 has written every (m_b, 1 / l_b)
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

// Shared-memory store of four words; async-proxy fence; TMA tile store and bulk groups.
__device__ __forceinline__ void m_st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void m_fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void m_tma_store_2d(const void *tmap, const void *src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void m_bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void m_bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void m_bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Work item q: row block nrb - 1 - q / n_maps of map q % n_maps.  The largest row blocks
// come first and a CTA's items (q = x, x + gridDim.x, ...) cover every row-block size,
// so the persistent CTAs get about the same number of tiles and the small items end the
// run.
__device__ __forceinline__ void m_item(int q, int n_maps, int nrb, int &map, int &rb) {
    map = q % n_maps;
    rb = nrb - 1 - q / n_maps;
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
                     const __grid_constant__ CUtensorMap tmO, const MapsParams p) {
    using C = MCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    MShared *sh = reinterpret_cast<MShared *>(smem + C::OFF_BAR);
    volatile int *abort = &sh->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // persistent: CTA x takes the items x, x + gridDim.x, ...; every role walks the same
    // items and counts tiles (g), so the pipelines run on across items
    const int n_items = p.n_maps * p.nrb;
    const int64_t lim = p.wait_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&sh->full[s], 1);
            mbar_init(&sh->empty[s], 1);
        }
        for (int s = 0; s < kMSBuf; ++s) {
            mbar_init(&sh->s_full[s], 1);
            mbar_init(&sh->s_empty[s], kMSoftmaxThreads);
        }
        for (int s = 0; s < 2; ++s) mbar_init(&sh->xch[s], kMSoftmaxThreads);
        for (int h = 0; h < kMParts; ++h) {
            mbar_init(&sh->stg_full[h], 4);  // one arrival per warp of the part
            mbar_init(&sh->stg_free[h], 1);  // the part's leader, once the store has read it
        }
        mbar_init(&sh->stat_ready, 128);
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
            int g = 0;
            for (int q = blockIdx.x; q < n_items && ok; q += gridDim.x) {
                int map, rb;
                m_item(q, p.n_maps, p.nrb, map, rb);
                const int nc = rb + 1, T = 2 * nc * p.B;
                for (int t = 0; t < T; ++t, ++g) {
                    const int st = g % C::NS;
                    if (g >= C::NS && !mbar_wait(&sh->empty[st], ((g / C::NS) - 1) & 1, lim, abort)) {
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
            }
            if (!ok) {
                report(p.status, SSA_ERR_TIMEOUT);
                *abort = 1;
            }
            // never leave the CTA with a copy still writing shared memory
            for (int u = (g > C::NS ? g - C::NS : 0); u < g; ++u)
                mbar_wait(&sh->full[u % C::NS], (u / C::NS) & 1, kMDrainNs, nullptr);
        }
    } else if (warp == kMWarpMma) {
        if (lane == 0) {
            // ------------------------------- MMA issuer -------------------------------
            // waits test the barrier first: try_wait in a thread with MMAs in flight costs
            // about their drain time even on a completed phase
            constexpr uint32_t IDESC = m_idesc(128, 128);
            bool ok = true;
            int n_tiles = 0;
            for (int q = blockIdx.x; q < n_items; q += gridDim.x) {
                int map, rb;
                m_item(q, p.n_maps, p.nrb, map, rb);
                n_tiles += 2 * (rb + 1) * p.B;
            }
            for (int g = 0; g < n_tiles && ok; ++g) {
                const int st = g % C::NS, sb = g % kMSBuf;
                if (!mbar_wait_poll(&sh->full[st], (g / C::NS) & 1, lim, abort)) ok = false;
                if (ok && g >= kMSBuf && !mbar_wait_poll(&sh->s_empty[sb], ((g / kMSBuf) - 1) & 1, lim, abort))
                    ok = false;
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
        const int h = warp >> 2;  // column part of every tile
        const int il = 32 * (warp & 3) + lane;
        int map = 0, rb = 0;  // the current item
        const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        float2 *stat = reinterpret_cast<float2 *>(smem + C::OFF_STAT);
        float2 *xch = reinterpret_cast<float2 *>(smem + C::OFF_XCH);  // [parity][part][row]
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2), zero2 = f2_pack(0.0f, 0.0f);
        float *row = p.maps;  // row 128 rb + il of the current item's map
        // A chunk of this part's columns of the row block (kMCols columns from col0), from
        // w of every thread.  Staged: each thread writes its row into the part's staging
        // buffer in the 128-byte swizzle the tensor map uses (16-byte unit j of row r at
        // j ^ (r % 8)), the warps report on stg_full, and the part's leader stores the box
        // with TMA and frees the buffer once the store has read it.
        const bool leader = (warp & 3) == 0 && lane == 0;
        uint8_t *stg = smem + C::OFF_STG + h * (128 * 128);
        int ne = 0;  // chunks written by this part
        auto put_chunk = [&](const uint32_t(&w)[kMCols], int col0) -> bool {
            if constexpr (C::STAGED) {
                if (ne >= 1 && !__all_sync(0xffffffffu, mbar_wait(&sh->stg_free[h], (ne - 1) & 1, lim, abort)))
                    return false;
                const uint32_t base = smem_u32(stg) + il * 128;
#pragma unroll
                for (int j = 0; j < kMCols / 4; ++j)
                    m_st_shared_v4(base + ((j ^ (il & 7)) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                m_fence_proxy_async();  // the generic-proxy writes, before the TMA reads them
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh->stg_full[h]);
                bool good = true;
                if (leader) {
                    if (mbar_wait(&sh->stg_full[h], ne & 1, lim, abort)) {
                        m_tma_store_2d(&tmO, stg, col0, map * p.L + 128 * rb);
                        m_bulk_commit();
                        m_bulk_wait_read();
                        mbar_arrive(&sh->stg_free[h]);
                    } else {
                        good = false;
                    }
                }
                ++ne;
                return __all_sync(0xffffffffu, good);
            } else {
                float *dst = row + col0;
                if (p.align32) {
#pragma unroll
                    for (int k = 0; k < kMCols / 8; ++k) st_global_v8(dst + 8 * k, w + 8 * k);
                } else {
#pragma unroll
                    for (int k = 0; k < kMCols / 4; ++k)
                        reinterpret_cast<uint4 *>(dst)[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                }
                return true;
            }
        };
        bool ok = true;
        float m = -INFINITY, l = 0.0f;
        uint64_t acc[kMCols / 2];  // the row's running sum over samples, packed pairs
#pragma unroll
        for (int k = 0; k < kMCols / 2; ++k) acc[k] = zero2;
        int g = 0, gb = 0, gi = 0;  // tiles, samples (pass-1 exchanges) and items so far
        for (int q = blockIdx.x; q < n_items && ok; q += gridDim.x, ++gi) {
            m_item(q, p.n_maps, p.nrb, map, rb);
            const int nc = rb + 1, T = 2 * nc * p.B;
            row = p.maps + (static_cast<size_t>(map) * p.L + 128 * rb + il) * p.L;
            for (int t = 0; t < T; ++t, ++g) {
                bool pass2;
                int b, c;
                m_tile(t, nc, p.B, pass2, b, c);
                const int sb = g % kMSBuf;
                if (pass2 && t == nc * p.B) {  // first tile of pass 2: every (m_b, 1 / l_b) is written
                    if (!__all_sync(0xffffffffu, mbar_wait(&sh->stat_ready, gi & 1, lim, abort))) {
                        ok = false;
                        break;
                    }
                }
                if (!__all_sync(0xffffffffu, mbar_wait(&sh->s_full[sb], (g / kMSBuf) & 1, lim, abort))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t r[kMCols];
                tmem_ld32(tmem + lane_off + 128 * sb + kMCols * h, r);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&sh->s_empty[sb]);  // the S buffer may take tile t + kMSBuf
                // causal keys of this row in the chunk: local column kMCols h + k < kv.  Only the
                // diagonal chunk (c == rb) masks; the warp-uniform test keeps the other chunks
                // free of selects.
                const bool diag = c == rb;
                const int kv = (diag ? il + 1 : 128) - kMCols * h;
                if (!pass2) {
                    uint64_t x[kMCols / 2];  // scaled logits as packed pairs (log2 domain)
#pragma unroll
                    for (int k = 0; k < kMCols / 2; ++k)
                        x[k] = f2_fma(f2_pack(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), sl2x2, zero2);
                    if (diag) {
#pragma unroll
                        for (int k = 0; k < kMCols / 2; ++k) {
                            float a, b2;
                            f2_unpack(x[k], a, b2);
                            x[k] = f2_pack(2 * k < kv ? a : -INFINITY, 2 * k + 1 < kv ? b2 : -INFINITY);
                        }
                    }
                    float mx[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float a, b2;
                        f2_unpack(x[q], a, b2);
                        mx[q] = fmaxf(a, b2);
                    }
#pragma unroll
                    for (int k = 4; k < kMCols / 2; ++k) {
                        float a, b2;
                        f2_unpack(x[k], a, b2);
                        mx[k & 3] = fmax3(mx[k & 3], a, b2);
                    }
                    const float m_new = fmaxf(m, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
                    if (m_new != -INFINITY) {  // else no causal key in this part yet
                        const uint64_t nm2 = f2_pack(-m_new, -m_new);
                        uint64_t sum[4] = {zero2, zero2, zero2, zero2};
#pragma unroll
                        for (int k = 0; k < kMCols / 2; ++k) {
                            float a, b2;
                            f2_unpack(f2_add(x[k], nm2), a, b2);
                            sum[k & 3] = f2_add(sum[k & 3], f2_pack(ex2_approx(a), ex2_approx(b2)));
                        }
                        float s0, s1, s2, s3, s4, s5, s6, s7;
                        f2_unpack(sum[0], s0, s1);
                        f2_unpack(sum[1], s2, s3);
                        f2_unpack(sum[2], s4, s5);
                        f2_unpack(sum[3], s6, s7);
                        l = l * ex2_approx(m - m_new) + (((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7)));
                        m = m_new;
                    }
                    if (c == nc - 1) {
                        // combine the parts of the row: every part computes the same
                        // (m_b, 1 / l_b) from the same pairs; part 0 keeps it for pass 2
                        // parts' slots double-buffered by sample parity: a part reaches the next
                        // exchange of the same parity only after everyone passed the one between
                        const int par = gb & 1;
                        xch[(par * kMParts + h) * 128 + il] = make_float2(m, l);
                        mbar_arrive(&sh->xch[par]);
                        if (!__all_sync(0xffffffffu, mbar_wait(&sh->xch[par], (gb >> 1) & 1, lim, abort))) {
                            ok = false;
                            break;
                        }
                        if (h == 0) {
                            float2 o[kMParts];
                            float mb = -INFINITY;
#pragma unroll
                            for (int q = 0; q < kMParts; ++q) {
                                o[q] = xch[(par * kMParts + q) * 128 + il];
                                mb = fmaxf(mb, o[q].x);  // finite: key 0 is causal for every row
                            }
                            float lb = 0.0f;
#pragma unroll
                            for (int q = 0; q < kMParts; ++q) lb += o[q].y * ex2_approx(o[q].x - mb);
                            stat[b * 128 + il] = make_float2(mb, 1.0f / lb);
                            if (b == p.B - 1) mbar_arrive(&sh->stat_ready);  // release: every stat written
                        }
                        m = -INFINITY;
                        l = 0.0f;
                        ++gb;
                    }
                } else {
                    const float2 st = stat[b * 128 + il];
                    const uint64_t nm2 = f2_pack(-st.x, -st.x), inv2 = f2_pack(st.y, st.y);
#pragma unroll
                    for (int k = 0; k < kMCols / 2; ++k) {
                        float a, b2;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), sl2x2, nm2), a,
                                  b2);
                        float e0 = ex2_approx(a), e1 = ex2_approx(b2);
                        if (diag) {
                            e0 = 2 * k < kv ? e0 : 0.0f;
                            e1 = 2 * k + 1 < kv ? e1 : 0.0f;
                        }
                        acc[k] = f2_fma(f2_pack(e0, e1), inv2, acc[k]);
                    }
                    if (b == p.B - 1) {
                        // the chunk of the map row, this part's columns
                        const uint64_t ib2 = f2_pack(p.inv_B, p.inv_B);
                        uint32_t w[kMCols];
#pragma unroll
                        for (int k = 0; k < kMCols / 2; ++k) {
                            float a, b2;
                            f2_unpack(f2_fma(acc[k], ib2, zero2), a, b2);
                            w[2 * k] = __float_as_uint(a);
                            w[2 * k + 1] = __float_as_uint(b2);
                            acc[k] = zero2;
                        }
                        if (!put_chunk(w, 128 * c + kMCols * h)) {
                            ok = false;
                            break;
                        }
                    }
                }
            }
            if (ok) {
                // the chunks above the diagonal block: zeros
                uint32_t z[kMCols];
#pragma unroll
                for (int k = 0; k < kMCols; ++k) z[k] = 0u;
                for (int cc = nc; cc < p.nrb && ok; ++cc) ok = put_chunk(z, 128 * cc + kMCols * h);
            }
        }
        if (!ok) {
            report(p.status, SSA_ERR_TIMEOUT);
            *abort = 1;
        }
        if (C::STAGED && leader) m_bulk_wait_all();  // every map store of the part complete
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

// 2-D map over the fp32 maps [n_maps * L rows][L columns]; box = 32 columns x 128 rows,
// 128-byte swizzle (the staging layout of the kernel).
int m_make_out_map(CUtensorMap *m, float *maps, int n_maps, int L) {
    auto enc = m_encode_fn();
    if (!enc) {
        set_error("cuTensorMapEncodeTiled is unavailable");
        return SSA_ERR_CUDA;
    }
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(n_maps) * L};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(L) * 4};
    cuuint32_t box[2] = {kMCols, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, maps, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) for the maps output (n_maps=%d L=%d)", static_cast<int>(r),
                  n_maps, L);
        return SSA_ERR_CUDA;
    }
    return SSA_OK;
}

template <int D>
int launch_maps(const void *Q, const void *K, const MapsParams &p, cudaStream_t s) {
    using C = MCfg<D>;
    CUtensorMap mQ, mK, mO;
    int rc;
    if ((rc = m_make_map(&mQ, Q, D, p.L, p.n_maps * p.B)) != SSA_OK) return rc;
    if ((rc = m_make_map(&mK, K, D, p.L, p.n_maps * p.B)) != SSA_OK) return rc;
    if ((rc = m_make_out_map(&mO, p.maps, p.n_maps, p.L)) != SSA_OK) return rc;
    SSA_CUDA_TRY(cudaFuncSetAttribute(attn_maps_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    int dev = 0, sms = 0;
    SSA_CUDA_TRY(cudaGetDevice(&dev));
    SSA_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const long long items = static_cast<long long>(p.n_maps) * p.nrb;
    const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);  // one persistent CTA per SM
    attn_maps_kernel<D><<<grid, kMThreads, C::SMEM, s>>>(mQ, mK, mO, p);
    SSA_LAUNCH_CHECK();
    return SSA_OK;
}

}  // namespace
}  // namespace ssa

using namespace ssa;

extern "C" int sparse_attn_maps(const void *Q, const void *K, int n_maps, int B, int L, int d, float scale,
                                float *maps, int32_t *dev_status, void *stream) {
    ssa::TraceRange trace_range("sparse_attn_maps");
    SSA_CHECK_ARG(Q && K && maps, "sparse_attn_maps: null pointer argument");
    if (d != 64 && d != 128) {
        set_error("sparse_attn_maps: head dimension must be 64 or 128 (got %d)", d);
        return SSA_ERR_UNSUPPORTED;
    }
    SSA_CHECK_ARG(n_maps >= 1 && B >= 1 && B <= kMapsMaxB, "sparse_attn_maps: need n_maps >= 1 and 1 <= B <= %d",
                  kMapsMaxB);
    SSA_CHECK_ARG(L >= 128 && L <= SSA_MAPS_MAX_L && L % 128 == 0,
                  "sparse_attn_maps: L must be a multiple of 128 in [128, %d] (got %d)", SSA_MAPS_MAX_L, L);
    // tile coordinates (sample index, map row) are 32-bit in the kernel and the TMA maps
    SSA_CHECK_ARG(static_cast<int64_t>(n_maps) * B < (1LL << 30) && static_cast<int64_t>(n_maps) * L < (1LL << 31),
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
