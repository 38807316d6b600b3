/*
 * ssa.h -- C ABI of libssa: DAM structured sparse attention on one B200 (sm_100a).
 *
 * The method is the Dynamic Attention Mask of the DAM review page ("DAM: Dynamic
 * Attention Mask for Long-Context Large Language Model Inference Acceleration",
 * pith review of arXiv 2506.11104):
 *   stage one  ("What carries the argument"): averaged L x L attention maps ->
 *              Box-Cox (lambda) -> threshold tau -> binary true mask M -> score every
 *              diagonal (j = i - r) and vertical (j = c, i >= c) candidate by
 *              gamma_k = sum(M P_k) / sum(P_k) -> keep gamma_k >= mu;
 *   stage two  ("What carries the argument"; "Circularity Check", steps 1 and 2;
 *              Referee Report summary): the kept patterns, pasted over S x S, form
 *              the extended mask applied to QK^T / sqrt(d_k) before the softmax.
 *
 * Conventions shared by every call
 *   - Every call returns an int status (SSA_OK or a negative SSA_ERR_* code) and
 *     records a message retrievable with ssa_last_error() (thread-local).
 *   - The caller owns all memory.  Every pointer argument named as "device" must
 *     point to CUDA device memory of the current device; "host" pointers to host
 *     memory.  The library allocates and frees nothing and never synchronises the
 *     stream, except where a call says so.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     All work of a call is enqueued on it, in order.
 *   - `dev_status` (device, one int32, may be NULL) receives faults detected on the
 *     GPU: the first non-zero SSA_ERR_* code written by any kernel stays.  The caller
 *     zeroes it and reads it after synchronising.  Kernels never trap: on a bad index
 *     or an expired bounded wait they record the code and return.
 *   - bf16 tensors are passed as raw 16-bit storage (uint16_t / void*).
 */
#ifndef SSA_H
#define SSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SSA_API __attribute__((visibility("default")))
#else
#define SSA_API
#endif

#define SSA_OK 0
#define SSA_ERR_INVALID (-1)     /* null pointer, bad size, unsorted/duplicate/negative list, bad map entry */
#define SSA_ERR_UNSUPPORTED (-2) /* head dim not 64/128, capture L > 1024, Case-2 plan given to decoding,
                                    a kernel build or device ordinal the library cannot use */
#define SSA_ERR_CAPACITY (-3)    /* caller buffer or workspace too small */
#define SSA_ERR_CUDA (-4)        /* a CUDA runtime/driver call failed */
#define SSA_ERR_TIMEOUT (-5)     /* a bounded on-device wait expired */

/* Tile edge of the query blocks and key tiles used by the plan and the kernels. */
#define SSA_BLOCK 128

/* ------------------------------------------------------------------------------ */
/* Stage one: averaged attention maps                                              */
/* ------------------------------------------------------------------------------ */

#define SSA_MAPS_MAX_B 32   /* samples averaged per call */
#define SSA_MAPS_MAX_L 4096

/*
 * sparse_attn_maps -- the averaged attention maps stage one starts from ("What carries
 * the argument": maps averaged over a calibration corpus; "Assumptions & free
 * parameters": capture length L = 512), produced on the GPU from B samples of each
 * map's query and key rows:
 *   maps[m][i][j] = (1/B) sum_b softmax_j( scale * Q[m][b][i] . K[m][b][j] )   j <= i
 *   maps[m][i][j] = 0                                                          j > i
 * (causal row softmax per sample, then the mean over the samples), in the layout
 * sparse_pattern_capture reads.  Arithmetic: bf16 inputs, fp32 logits (tensor cores),
 * fp32 softmax with hardware 2^x, fp32 mean; each row sums to 1 up to fp32 rounding.
 *
 *   Q, K     device, bf16 [n_maps][B][L][d] contiguous (sample b of map m at
 *            (m * B + b) * L * d), 16-byte aligned
 *   n_maps   >= 1 with n_maps * L < 2^31 and n_maps * B < 2^30;  B in [1, SSA_MAPS_MAX_B];
 *            L a multiple of 128 in [128, SSA_MAPS_MAX_L]
 *   d        64 or 128 (else SSA_ERR_UNSUPPORTED)
 *   scale    > 0, usually 1 / sqrt(d)
 *   maps     device, float32 [n_maps][L][L] row-major, 16-byte aligned; every entry
 *            is written
 * Errors: SSA_ERR_INVALID for a null or misaligned pointer or a size out of range; an
 * expired bounded wait sets SSA_ERR_TIMEOUT in dev_status (maps then unspecified).
 * For B larger than SSA_MAPS_MAX_B, average the maps of several calls weighted by
 * their sample counts.
 */
SSA_API int sparse_attn_maps(const void *Q, const void *K, int n_maps, int B, int L, int d, float scale,
                             float *maps, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------------ */
/* Stage one: pattern capture                                                      */
/* ------------------------------------------------------------------------------ */

/* Workspace bytes sparse_pattern_capture needs for n_maps maps of size L x L. */
SSA_API size_t sparse_pattern_capture_ws_bytes(int n_maps, int L);

/*
 * sparse_pattern_capture -- stage one of DAM ("What carries the argument"; lambda,
 * tau, mu from "Assumptions & free parameters"; eps from Referee Report minor
 * comment 1).
 *
 * For every map m and row i (causal entries j <= i only):
 *   y_j = ((x_j + eps)^lambda - 1) / lambda                (Box-Cox)
 *   t_j = (y_j - y_min) / (y_max - y_min)  (row min/max; t = 1 on a constant row)
 *   M[i][j] = t_j >= tau
 * then gamma_diag[r] = #{i >= r : M[i][i-r]} / (L - r), gamma_vert[c] =
 * #{i >= c : M[i][c]} / (L - c), both in fp64, and r (resp. c) is kept iff
 * gamma >= mu.  At lambda 0.5 and 1 every threshold decision is made with correctly
 * rounded fp64 arithmetic in the stated order, so the kept lists are exactly
 * reproducible.  Other lambdas (0 = log) go through fp64 pow / log, which are not
 * correctly rounded: an entry whose t lies within a few units in the last place of
 * tau may be decided differently by another implementation.
 *
 *   maps         device, float32 [n_maps][L][L] row-major, already averaged over the
 *                calibration batches; causal entries must be finite and >= 0
 *                (entries j > i are ignored)
 *   n_maps       >= 1;  L in [1, 1024]
 *   lambda       in [0, 64] (else SSA_ERR_INVALID); tau, mu in fp64; eps >= 0
 *   diag_ptr     device int32 [n_maps + 1]   CSR row pointers of the kept diagonals
 *   diag_offsets device int32 [n_maps * L]   kept r, ascending within each map
 *   vert_ptr     device int32 [n_maps + 1]
 *   vert_cols    device int32 [n_maps * L]   kept c, ascending within each map
 *   ws           device workspace of at least sparse_pattern_capture_ws_bytes()
 * A negative or non-finite map entry sets SSA_ERR_INVALID in dev_status; the lists
 * are then unspecified.  When maps is 16-byte aligned and L a multiple of 4, rows are
 * staged into shared memory by bulk copies whose waits are bounded
 * (ssa_set_wait_limit_ns): an expired wait sets SSA_ERR_TIMEOUT in dev_status, the
 * kernel waits (again bounded) for its copies in flight and the lists are unspecified.
 */
SSA_API int sparse_pattern_capture(const float *maps, int n_maps, int L, double lambda, double tau,
                           double mu, double eps, int32_t *diag_ptr, int32_t *diag_offsets,
                           int32_t *vert_ptr, int32_t *vert_cols, void *ws, size_t ws_bytes,
                           int32_t *dev_status, void *stream);

/* Scalings of the Box-Cox output to [0, 1] before tau (the page leaves it unstated). */
#define SSA_SCALE_ROW 0 /* min and max over each row's causal entries (the default reading) */
#define SSA_SCALE_MAP 1 /* min and max over all causal entries of the map */

/*
 * sparse_pattern_capture_ex -- sparse_pattern_capture with the two optional readings
 * and outputs of stage one:
 *   scaling    SSA_SCALE_ROW (as sparse_pattern_capture) or SSA_SCALE_MAP: every row
 *              of a map uses the map's min and max (a constant map has t = 1); this
 *              reading reads the maps twice (a min/max pass, then the decisions)
 *   true_mask  null, or device uint32 [n_maps][L][ceil(L/32)], 4-byte aligned: the
 *              binary true mask M itself, bit (j % 32) of word j / 32 of row i set iff
 *              j <= i and M[i][j] (the input of the Case-2 extension,
 *              sparse_pattern_extend_case2)
 * All other arguments, the workspace and the errors are those of
 * sparse_pattern_capture; a scaling other than the two is SSA_ERR_INVALID.
 */
SSA_API int sparse_pattern_capture_ex(const float *maps, int n_maps, int L, double lambda, double tau,
                                      double mu, double eps, int scaling, int32_t *diag_ptr,
                                      int32_t *diag_offsets, int32_t *vert_ptr, int32_t *vert_cols,
                                      uint32_t *true_mask, void *ws, size_t ws_bytes,
                                      int32_t *dev_status, void *stream);

/* Size of the fixed device scratch of sparse_pattern_capture_noalloc (8 MiB). */
#define SSA_CAPTURE_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * sparse_pattern_capture_noalloc -- sparse_pattern_capture without a workspace
 * argument.  The paper has no counterpart: this is a deployment variant.
 *
 * For callers that cannot allocate device memory: a plugin host that only hands the
 * library its input and output buffers and has no allocator to lend, or a serving
 * process that must not call cudaMalloc/cudaFree after start-up because those calls
 * can synchronise the device and stall every other stream.  The call itself allocates
 * nothing: its scratch is a fixed SSA_CAPTURE_NOALLOC_SCRATCH_BYTES device array
 * inside the library, held by every GPU that loads the library until the process
 * exits.  Arguments, outputs and results are those of sparse_pattern_capture; the
 * caller still provides maps, the four output lists and dev_status.
 *
 *   - Sizes whose scratch (sparse_pattern_capture_ws_bytes(n_maps, L)) exceeds the
 *     fixed size are rejected with SSA_ERR_CAPACITY before any device work
 *     (L = 512 allows up to 1023 maps).
 *   - The first call on each device looks up the array's device address with that
 *     device current and keeps it for the life of the process; make that first call
 *     before any stream capture begins.  A device reset (cudaDeviceReset, or anything
 *     else that tears down the primary context) invalidates the kept address: do not
 *     call this entry point again in a process that has reset the device.
 *   - Every call shares the one array per device and clears what must start at zero
 *     itself; calls that overlap on the GPU (different streams or host threads) race
 *     on it and must be serialised by the caller.
 */
SSA_API int sparse_pattern_capture_noalloc(const float *maps, int n_maps, int L, double lambda,
                                           double tau, double mu, double eps, int32_t *diag_ptr,
                                           int32_t *diag_offsets, int32_t *vert_ptr,
                                           int32_t *vert_cols, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------------ */
/* Stage two: extension to S and the tile plan                                     */
/* ------------------------------------------------------------------------------ */

/* Sizes of a plan, filled by the sizing pass of sparse_pattern_extend. */
typedef struct ssa_plan_sizes {
    int32_t n_heads;
    int32_t S;
    int32_t nqb;       /* ceil(S / 128) */
    int32_t n_diag;    /* total extended diagonals over all heads */
    int32_t n_vert;    /* total extended columns over all heads */
    int32_t max_vert;  /* max over heads of the extended column count */
    int64_t n_tiles;   /* total listed band tiles */
    int32_t bitmap_slots; /* Case-2 plans: element-bitmap slots per head (0 otherwise) */
} ssa_plan_sizes;

/*
 * A compiled plan.  The struct itself is host memory; every pointer in it is a
 * device buffer owned by the caller and sized from ssa_plan_sizes:
 *   ext_diag_ptr [n_heads+1], ext_diag_offsets [max(n_diag,1)],
 *   ext_vert_ptr [n_heads+1], ext_vert_cols [max(n_vert,1)],
 *   tile_ptr [n_heads*nqb + 1], tile_key0 [max(n_tiles,1)],
 *   tile_dmask [max(n_tiles,1)][4] (uint64), tile_cmask [max(n_tiles,1)][2] (uint64),
 *   tile_flags [max(n_tiles,1)], stripe_cnt [n_heads*nqb].
 * Tile semantics, for head h and query block qb (rows lo = 128qb .. hi = 128qb+127):
 *   needed keys: j in [0, hi] such that some extended diagonal r has lo-j <= r <= hi-j
 *   (all 128 rows count, even in a ragged last block); the band tiles are key windows
 *   key0 .. key0+127, chosen greedily: the first starts at the smallest needed key,
 *   each next one at the smallest needed key >= previous key0 + 128 (so a band whose
 *   keys do not start at a multiple of 128 still takes ceil(width / 128) windows);
 *   dmask bit t (0..254) set  iff  r = 128qb - key0 + t - 127 is an extended diagonal
 *   cmask bit jl (0..127) set iff  column key0 + jl is an extended column
 *   a window is listed, in ascending key0, iff some (i, j) in it has i < S,
 *   i - j a diagonal and j not a column; tile_flags bit 0 (FULL) iff 128(qb+1) <= S,
 *   all 255 dmask bits set and cmask == 0;
 *   stripe_cnt[h*nqb+qb] = #{extended columns c <= min(S-1, 128qb+127)}.
 * The windows are disjoint and cover every needed key, and columns are owned by the
 * stripe phase only, so each retained pair is used once.
 */
typedef struct ssa_plan {
    int32_t n_heads;
    int32_t S;
    int32_t nqb;
    int32_t max_vert;
    int64_t n_tiles; /* capacity of the tile arrays (from ssa_plan_sizes) */
    int32_t *ext_diag_ptr;
    int32_t *ext_diag_offsets;
    int32_t *ext_vert_ptr;
    int32_t *ext_vert_cols;
    int32_t *tile_ptr;
    int32_t *tile_key0;
    uint64_t *tile_dmask;
    uint64_t *tile_cmask;
    uint32_t *tile_flags;
    int32_t *stripe_cnt;
    /* Case-2 plans only (sparse_pattern_extend_case2; zero / NULL otherwise): */
    int32_t bitmap_slots; /* from ssa_plan_sizes */
    uint64_t *tile_bits;  /* [n_heads * bitmap_slots][128][2] (uint64), 16-byte aligned */
    /* Capacities of ext_diag_offsets and ext_vert_cols (n_diag, n_vert from
     * ssa_plan_sizes).  A fill pass whose extended lists need more (in total, or more
     * than max_vert columns for one head) changes nothing in the plan and reports
     * SSA_ERR_CAPACITY in dev_status; the tile arrays are checked against n_tiles the
     * same way. */
    int32_t n_diag;
    int32_t n_vert;
} ssa_plan;

/* Workspace bytes of either pass of sparse_pattern_extend (about 4 * n_heads * S for
 * the per-diagonal run starts, plus small per-block counters). */
SSA_API size_t sparse_pattern_extend_ws_bytes(int n_heads, int S);

/*
 * sparse_pattern_extend -- stage two of DAM ("What carries the argument": the kept
 * patterns are pasted into an S x S mask; "Circularity Check" step 1: that mask is
 * the union of the matched patterns).  The extended lists keep every diagonal r < S
 * and column c < S of each head; the plan then lists, per query block, the key tiles
 * the band touches.
 *
 *   n_heads, S   >= 1
 *   diag_ptr, diag_offsets, vert_ptr, vert_cols
 *                device CSR lists per head (e.g. the output of capture); each list
 *                strictly ascending and >= 0, else SSA_ERR_INVALID
 *   sizes        host, always filled when plan == NULL (sizing pass)
 *   plan         NULL: sizing pass -- enqueues the counting kernels, copies the
 *                totals to the host and SYNCHRONISES `stream`; returns
 *                SSA_ERR_INVALID if a list is malformed, SSA_ERR_CAPACITY if the plan
 *                would hold more than INT32_MAX tiles (tile_ptr is int32).
 *                non-NULL: fill pass -- writes every plan array (no synchronisation);
 *                the new lists and tiles are counted in the workspace first, and only
 *                when they fit the plan's capacities (n_diag, n_vert, max_vert,
 *                n_tiles) is the plan written; otherwise it keeps its previous content
 *                and SSA_ERR_CAPACITY goes to dev_status.  plan->n_heads/S/nqb must
 *                match the call.
 *   ws           device workspace of at least sparse_pattern_extend_ws_bytes()
 */
SSA_API int sparse_pattern_extend(int n_heads, const int32_t *diag_ptr, const int32_t *diag_offsets,
                          const int32_t *vert_ptr, const int32_t *vert_cols, int S,
                          ssa_plan_sizes *sizes, const ssa_plan *plan, void *ws, size_t ws_bytes,
                          int32_t *dev_status, void *stream);

/*
 * sparse_pattern_extend_case2 -- the Case-2 reading of the extension (DAM review page,
 * Referee Report major comment 2: the patterns are pasted beyond the first L tokens):
 * the captured L x L true mask of each head is kept verbatim in the first block, the
 * union of the kept patterns everywhere else.  Cell (i, j), j <= i < S, is retained iff
 *   i < L:  bit j of row i of true_mask[h]     (the patterns play no part there)
 *   i >= L: i - j is a kept diagonal or j a kept column (as sparse_pattern_extend).
 * The paper has no tile plan; this is the library's layout: every query block holding
 * a row below min(L, S) is covered by element-bitmap tiles, one per key block kb = 0..qb
 * (key0 = 128 kb), listed when any of its cells is set, with tile_flags bit 1 (BITMAP),
 * the bitmap's slot h * bitmap_slots + qb (qb + 1) / 2 + kb in tile_dmask word 0, and
 * no stripe tiles (stripe_cnt 0); plan->tile_bits[slot][il][w] holds the cells of row il,
 * key column jl at bit jl % 64 of word jl / 64.  The other query blocks have the plan of
 * sparse_pattern_extend.
 *
 *   true_mask  device uint32 [n_heads][L][ceil(L/32)], 4-byte aligned, bit j % 32 of
 *              word j / 32 of row i = M[i][j] (sparse_pattern_capture_ex writes it;
 *              bits above the diagonal are ignored)
 *   L          capture length, [1, 1024]
 * Everything else as sparse_pattern_extend; the sizing pass also sets
 * sizes->bitmap_slots, and the fill pass needs plan->bitmap_slots equal to it and
 * plan->tile_bits (16-byte aligned) of n_heads * bitmap_slots * 128 * 2 uint64.
 * sparse_attn_fwd takes the plan as it is; sparse_attn_decode rejects it
 * (SSA_ERR_UNSUPPORTED: decoding follows the first reading only).
 */
SSA_API int sparse_pattern_extend_case2(int n_heads, const int32_t *diag_ptr, const int32_t *diag_offsets,
                                        const int32_t *vert_ptr, const int32_t *vert_cols,
                                        const uint32_t *true_mask, int L, int S, ssa_plan_sizes *sizes,
                                        const ssa_plan *plan, void *ws, size_t ws_bytes, int32_t *dev_status,
                                        void *stream);

/* ------------------------------------------------------------------------------ */
/* Attention forward                                                               */
/* ------------------------------------------------------------------------------ */

/* Workspace bytes of sparse_attn_fwd: a 256-byte work counter followed by the
 * gathered stripe keys and values. */
SSA_API size_t sparse_attn_fwd_ws_bytes(int n_heads, int max_vert, int d);

/*
 * sparse_attn_fwd -- causal prefill attention restricted to the extended mask
 * (Referee Report summary and "Circularity Check" step 2: the mask is applied to
 * QK^T / sqrt(d_k) before the softmax; "What carries the argument": only the
 * retained connections are computed).  For head h, KV head g = kv_map[h] (or
 * h / (H_q/H_kv) when kv_map is NULL) and query i < S, with retained keys
 * J_i = {i - r : r in D_h, r <= i} U {c in C_h : c <= i}:
 *   O[h][i]   = sum_{j in J_i} softmax_j(scale * q_i . k_j) v_j
 *   LSE[h][i] = log sum_{j in J_i} exp(scale * q_i . k_j)     (natural log)
 * An empty J_i gives O = 0 and LSE = -inf.  bf16 inputs, fp32 accumulation, bf16 O.
 *
 *   Q, O         device bf16 [H_q][S][d], contiguous
 *   K, V         device bf16 [H_kv][S][d], contiguous
 *   H_q, H_kv    >= 1; H_q % H_kv == 0 when kv_map is NULL
 *   S            must equal plan->S;  d in {64, 128} (else SSA_ERR_UNSUPPORTED)
 *   plan         host struct of device arrays from sparse_pattern_extend, n_heads == H_q
 *   kv_map       device int32 [H_q] or NULL; entries outside [0, H_kv) set
 *                SSA_ERR_INVALID in dev_status
 *   scale        softmax scale (1/sqrt(d) for the paper's formula)
 *   LSE          device float32 [H_q][S]
 *   ws           device workspace of at least sparse_attn_fwd_ws_bytes(H_q, plan->max_vert, d);
 *                all base pointers must be 16-byte aligned
 */
SSA_API int sparse_attn_fwd(const void *Q, const void *K, const void *V, int H_q, int H_kv, int S, int d,
                    const ssa_plan *plan, const int32_t *kv_map, float scale, void *O, float *LSE,
                    void *ws, size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------------ */
/* Decoding step                                                                   */
/* ------------------------------------------------------------------------------ */

/* Workspace bytes of sparse_attn_decode: the per-split partial results
 * ((2 + d) floats per split, 1 to 16 splits per sequence and head). */
SSA_API size_t sparse_attn_decode_ws_bytes(int B, int H_q, int d);

/*
 * sparse_attn_decode -- one decoding step over the same extended mask: the new query
 * of sequence b sits at position pos[b] and attends to row pos[b] of the mask ("What
 * carries the argument": the kept patterns are pasted over the whole S x S square;
 * Referee Report summary: the mask is applied to the scaled logits before the
 * softmax), i.e. for head h with KV head g:
 *   J = {pos - r : r an extended diagonal, r <= pos} U {c an extended column, c <= pos}
 *   O[b][h]   = sum_{j in J} softmax_j(scale * q . K[b][g][j]) V[b][g][j]
 *   LSE[b][h] = log sum_{j in J} exp(scale * q . K[b][g][j])      (natural log)
 * which is row pos[b] of sparse_attn_fwd over the same cache.  An empty J gives O = 0
 * and LSE = -inf.  bf16 inputs, fp32 accumulation, bf16 O.  Bound by the HBM traffic
 * of the gathered key and value rows.
 *
 *   Q, O         device bf16 [B][H_q][d], contiguous
 *   K, V         device bf16 [B][H_kv][S_cache][d]: the key/value cache of each sequence
 *   B, H_q, H_kv >= 1 (B, H_q <= 65535); H_q % H_kv == 0 when kv_map is NULL
 *   S_cache      must equal plan->S;  d in {64, 128} (else SSA_ERR_UNSUPPORTED)
 *   pos          device int32 [B], 0 <= pos[b] < S_cache; a position outside that range
 *                (or a kv_map entry outside [0, H_kv)) sets SSA_ERR_INVALID in
 *                dev_status and gives that sequence O = 0, LSE = -inf
 *   plan         from sparse_pattern_extend with S = S_cache and n_heads = H_q (only its
 *                extended lists are read)
 *   LSE          device float32 [B][H_q]
 *   ws           device workspace of at least sparse_attn_decode_ws_bytes(B, H_q, d);
 *                Q, K, V, O and ws 16-byte aligned
 */
SSA_API int sparse_attn_decode(const void *Q, const void *K, const void *V, int B, int H_q, int H_kv,
                               int S_cache, int d, const int32_t *pos, const ssa_plan *plan,
                               const int32_t *kv_map, float scale, void *O, float *LSE, void *ws,
                               size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------------ */
/* Diagnostics                                                                     */
/* ------------------------------------------------------------------------------ */

/* Message of the last failing call on this thread ("" if none). */
SSA_API const char *ssa_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
SSA_API int ssa_version(void);

/*
 * Time limit, in nanoseconds, of every bounded wait inside the kernels that wait on
 * copies or tensor-core work (attention, averaged maps, capture; default 2e9; 0 makes a
 * wait give up at its first unsuccessful poll).  When a wait expires the kernel writes
 * SSA_ERR_TIMEOUT to dev_status, drains its own copies and tensor-core work in flight,
 * frees its tensor memory and returns.  Process-wide; meant for fault-handling tests.
 * Returns the previous value.
 */
SSA_API int64_t ssa_set_wait_limit_ns(int64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H */
