/*
 * ssa_oracle.c -- plain, slow, obviously correct CPU oracle for DAM structured sparse
 * attention.  TEST INFRASTRUCTURE ONLY: it is built and called by the tests, by the
 * smoke check and by the benchmark's CPU-baseline leg, never by the library itself.
 * It shares no code, header or constant generator with the CUDA path.
 *
 * Source of every definition: the DAM review page, "DAM: Dynamic Attention Mask for
 * Long-Context Large Language Model Inference Acceleration" (pith review of arXiv
 * 2506.11104):
 *   - "What carries the argument": capture length L, Box-Cox with lambda, threshold
 *     tau to a binary true mask M, pattern pool of diagonals (j = i - r) and verticals
 *     (j = c, i >= c), score gamma_k = sum(M*P_k)/sum(P_k), keep gamma_k >= mu, paste
 *     the kept patterns into an S x S mask applied to the logits before softmax.
 *   - "Circularity Check", step 1: the pool is the union of the diagonal and vertical
 *     sets, and the extended mask is the sum (union) of the matched patterns.
 *   - "Circularity Check", step 2 and the Referee Report summary: the mask is applied
 *     to QK^T / sqrt(d_k) before softmax.
 *   - Referee Report, minor comment 1: the stabiliser eps (1e-8 in the main text).
 * Readings where the page is silent: row-wise
 * min-max scaling of the Box-Cox output before tau (map-wise as an option); t >= tau
 * and gamma >= mu; a constant row (or map) counts as t = 1; masked logits are excluded from the softmax (-inf),
 * not multiplied by 0; an empty row gives O = 0 and LSE = -inf; LSE is the natural
 * log-sum-exp of the scaled logits.
 *
 * Parity status: capture follows the readings above (the page gives no worked example,
 * so which min-max reading the paper used is "parity unpinned" against the paper; the
 * arithmetic of both is pinned by closed forms, hand-derived masks and invariants in
 * the tests).
 *
 * All floating point is IEEE binary64, built with -ffp-contract=off (no FMA fusion).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_OK 0
#define ORA_ERR_INVALID (-1)
#define ORA_ERR_CAPACITY (-3)
#define ORA_ERR_NOMEM (-6)

/* Tile edge of the canonical tile plan (the plan's own definition, not the paper's). */
#define ORA_TILE 128

static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ----------------------------------------------------------------------------------
 * Stage one: true mask, gamma scores, selection
 * -------------------------------------------------------------------------------- */

/* Box-Cox transform (Box & Cox 1964) of v + eps: ((v+eps)^lambda - 1) / lambda, and
 * log(v+eps) at lambda = 0.  lambda = 0.5 uses sqrt (exactly the square root). */
static double box_cox(double v, double lambda, double eps) {
    double z = v + eps;
    if (lambda == 0.0) return log(z);
    if (lambda == 0.5) return (sqrt(z) - 1.0) / lambda;
    if (lambda == 1.0) return (z - 1.0) / lambda;
    return (pow(z, lambda) - 1.0) / lambda;
}

/* True mask of one L x L averaged attention map (row-major float32), with the Box-Cox
 * output scaled to [0,1] before the threshold (the page does not say how; two readings):
 *   scaling 0 (per row): row i uses the min and max of its own causal entries j <= i;
 *   scaling 1 (per map): every row uses the min and max over all causal entries of the
 *                        map.
 * Then M[i][j] = (t >= tau) for j <= i, where t = (bc(x) - bc(min)) / (bc(max) - bc(min))
 * and t = 1 when max == min.  Entries j > i are 0. */
int ora_true_mask_ex(const float *map, int L, double lambda, double eps, double tau, int scaling,
                     uint8_t *M) {
    if (!map || !M || L <= 0 || (scaling != 0 && scaling != 1)) return ORA_ERR_INVALID;
    double map_mn = INFINITY, map_mx = -INFINITY;
    for (int i = 0; i < L; ++i)
        for (int j = 0; j <= i; ++j) {
            double x = (double)map[(size_t)i * L + j];
            if (x < map_mn) map_mn = x;
            if (x > map_mx) map_mx = x;
        }
    for (int i = 0; i < L; ++i) {
        const float *row = map + (size_t)i * L;
        double mn = INFINITY, mx = -INFINITY;
        for (int j = 0; j <= i; ++j) {
            double x = (double)row[j];
            if (x < mn) mn = x;
            if (x > mx) mx = x;
        }
        if (scaling == 1) {
            mn = map_mn;
            mx = map_mx;
        }
        double ylo = box_cox(mn, lambda, eps);
        double yhi = box_cox(mx, lambda, eps);
        for (int j = 0; j < L; ++j) {
            uint8_t bit = 0;
            if (j <= i) {
                double t;
                if (mx == mn) {
                    t = 1.0;
                } else {
                    t = (box_cox((double)row[j], lambda, eps) - ylo) / (yhi - ylo);
                }
                bit = (t >= tau) ? 1 : 0;
            }
            M[(size_t)i * L + j] = bit;
        }
    }
    return ORA_OK;
}

/* The per-row reading (scaling 0). */
int ora_true_mask(const float *map, int L, double lambda, double eps, double tau, uint8_t *M) {
    return ora_true_mask_ex(map, L, lambda, eps, tau, 0, M);
}

/* gamma_k = sum_{i,j} M[i][j] P_k[i][j] / sum_{i,j} P_k[i][j], with the sums taken over
 * the cells of pattern k: diagonal r covers (i, i-r) for i in [r, L); vertical c covers
 * (i, c) for i in [c, L). */
int ora_gamma(const uint8_t *M, int L, double *gamma_diag, double *gamma_vert) {
    if (!M || L <= 0) return ORA_ERR_INVALID;
    for (int r = 0; r < L; ++r) {
        long num = 0, den = 0;
        for (int i = r; i < L; ++i) {
            num += M[(size_t)i * L + (i - r)];
            den += 1;
        }
        gamma_diag[r] = (double)num / (double)den;
    }
    for (int c = 0; c < L; ++c) {
        long num = 0, den = 0;
        for (int i = c; i < L; ++i) {
            num += M[(size_t)i * L + c];
            den += 1;
        }
        gamma_vert[c] = (double)num / (double)den;
    }
    return ORA_OK;
}

/* Keep every candidate with gamma >= mu, in ascending order of r (resp. c). */
int ora_select(const double *gamma_diag, const double *gamma_vert, int L, double mu,
               int32_t *diag_out, int32_t *n_diag, int32_t *vert_out, int32_t *n_vert) {
    int nd = 0, nv = 0;
    for (int r = 0; r < L; ++r)
        if (gamma_diag[r] >= mu) diag_out[nd++] = r;
    for (int c = 0; c < L; ++c)
        if (gamma_vert[c] >= mu) vert_out[nv++] = c;
    *n_diag = nd;
    *n_vert = nv;
    return ORA_OK;
}

/* Whole stage one over n_maps maps [n_maps][L][L] with the given scaling (see
 * ora_true_mask_ex); outputs are CSR lists per map with capacity n_maps*L each
 * (diag_ptr / vert_ptr have n_maps+1 entries). */
int ora_capture_ex(const float *maps, int n_maps, int L, double lambda, double tau, double mu,
                   double eps, int scaling, int32_t *diag_ptr, int32_t *diag_offsets,
                   int32_t *vert_ptr, int32_t *vert_cols) {
    if (!maps || n_maps < 0 || L <= 0 || (scaling != 0 && scaling != 1)) return ORA_ERR_INVALID;
    int32_t *tmp_d = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_maps * L + 4);
    int32_t *tmp_v = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_maps * L + 4);
    int32_t *cnt_d = (int32_t *)calloc((size_t)n_maps + 1, sizeof(int32_t));
    int32_t *cnt_v = (int32_t *)calloc((size_t)n_maps + 1, sizeof(int32_t));
    int err = ORA_OK;
    if (!tmp_d || !tmp_v || !cnt_d || !cnt_v) err = ORA_ERR_NOMEM;
    if (err == ORA_OK) {
#pragma omp parallel
        {
            uint8_t *M = (uint8_t *)malloc((size_t)L * L);
            double *gd = (double *)malloc(sizeof(double) * (size_t)L);
            double *gv = (double *)malloc(sizeof(double) * (size_t)L);
#pragma omp for schedule(dynamic, 1)
            for (int m = 0; m < n_maps; ++m) {
                if (!M || !gd || !gv) continue;
                ora_true_mask_ex(maps + (size_t)m * L * L, L, lambda, eps, tau, scaling, M);
                ora_gamma(M, L, gd, gv);
                ora_select(gd, gv, L, mu, tmp_d + (size_t)m * L, &cnt_d[m], tmp_v + (size_t)m * L,
                           &cnt_v[m]);
            }
            if (!M || !gd || !gv) err = ORA_ERR_NOMEM;
            free(M);
            free(gd);
            free(gv);
        }
    }
    if (err == ORA_OK) {
        diag_ptr[0] = 0;
        vert_ptr[0] = 0;
        for (int m = 0; m < n_maps; ++m) {
            memcpy(diag_offsets + diag_ptr[m], tmp_d + (size_t)m * L, sizeof(int32_t) * cnt_d[m]);
            memcpy(vert_cols + vert_ptr[m], tmp_v + (size_t)m * L, sizeof(int32_t) * cnt_v[m]);
            diag_ptr[m + 1] = diag_ptr[m] + cnt_d[m];
            vert_ptr[m + 1] = vert_ptr[m] + cnt_v[m];
        }
    }
    free(tmp_d);
    free(tmp_v);
    free(cnt_d);
    free(cnt_v);
    return err;
}

/* The per-row reading (scaling 0). */
int ora_capture(const float *maps, int n_maps, int L, double lambda, double tau, double mu,
                double eps, int32_t *diag_ptr, int32_t *diag_offsets, int32_t *vert_ptr,
                int32_t *vert_cols) {
    return ora_capture_ex(maps, n_maps, L, lambda, tau, mu, eps, 0, diag_ptr, diag_offsets, vert_ptr,
                          vert_cols);
}

/* ----------------------------------------------------------------------------------
 * Stage two: extension of the kept patterns to S x S
 * -------------------------------------------------------------------------------- */

static int list_ok(const int32_t *a, int n) {
    for (int k = 0; k < n; ++k) {
        if (a[k] < 0) return 0;
        if (k > 0 && a[k] <= a[k - 1]) return 0;
    }
    return 1;
}

/* Extended mask over S x S = union of the kept patterns pasted at every causal
 * position; in list form that keeps each diagonal r < S and each column c < S. */
int ora_extend(int n_heads, const int32_t *diag_ptr, const int32_t *diag_offsets,
               const int32_t *vert_ptr, const int32_t *vert_cols, int S, int32_t *ext_diag_ptr,
               int32_t *ext_diag_offsets, int32_t *ext_vert_ptr, int32_t *ext_vert_cols) {
    if (n_heads < 0 || S <= 0) return ORA_ERR_INVALID;
    ext_diag_ptr[0] = 0;
    ext_vert_ptr[0] = 0;
    for (int h = 0; h < n_heads; ++h) {
        const int32_t *D = diag_offsets + diag_ptr[h];
        int nd = diag_ptr[h + 1] - diag_ptr[h];
        const int32_t *C = vert_cols + vert_ptr[h];
        int nc = vert_ptr[h + 1] - vert_ptr[h];
        if (nd < 0 || nc < 0 || !list_ok(D, nd) || !list_ok(C, nc)) return ORA_ERR_INVALID;
        int od = ext_diag_ptr[h], oc = ext_vert_ptr[h];
        for (int k = 0; k < nd; ++k)
            if (D[k] < S) ext_diag_offsets[od++] = D[k];
        for (int k = 0; k < nc; ++k)
            if (C[k] < S) ext_vert_cols[oc++] = C[k];
        ext_diag_ptr[h + 1] = od;
        ext_vert_ptr[h + 1] = oc;
    }
    return ORA_OK;
}

/* ----------------------------------------------------------------------------------
 * Canonical tile plan (this library's own layout of the extended mask).  For head h
 * and query block qb (rows lo = 128qb .. hi = 128qb + 127; rows >= S hold no pair):
 *   needed keys      j in [0, hi] such that some r in D_h has lo - j <= r <= hi - j
 *                    (the keys some diagonal reaches from some row of the block,
 *                    counting all 128 rows even in a ragged last block)
 *   key windows      greedy: the first starts at the smallest needed key, each next
 *                    one at the smallest needed key >= (previous start + 128); a
 *                    window with start key0 covers keys key0 .. key0 + 127
 *   dmask bit t (0..254) set  iff  r = 128qb - key0 + t - 127 is in D_h
 *   cmask bit jl (0..127) set iff  key0 + jl is in C_h
 *   a window is listed (ascending key0) iff some (i, j) of it has i < S,
 *                    i - j in D_h and j not in C_h (j <= i follows from r >= 0)
 *   FULL flag (bit 0)         iff  128(qb+1) <= S, all 255 dmask bits set and
 *                                  cmask == 0
 *   stripe_cnt[h][qb]          =   #{c in C_h : c <= min(S-1, 128qb+127)}
 * The windows are disjoint and cover every needed key, so each retained pair of the
 * band lies in exactly one listed window.  Two independent routines compute the
 * plan; the tests require them to agree.
 * -------------------------------------------------------------------------------- */

static void set_bit(uint64_t *w, int b) { w[b >> 6] |= (uint64_t)1 << (b & 63); }
static int get_bit(const uint64_t *w, int b) { return (int)((w[b >> 6] >> (b & 63)) & 1u); }

static int popcount256(const uint64_t *w) {
    int n = 0;
    for (int k = 0; k < 4; ++k) {
        uint64_t x = w[k];
        while (x) {
            x &= x - 1;
            ++n;
        }
    }
    return n;
}

static int32_t count_le(const int32_t *a, int n, int32_t x) {
    int c = 0;
    for (int k = 0; k < n; ++k)
        if (a[k] <= x) ++c;
    return c;
}

/* Routine 1: brute force over every (i, j) of the block (small S only).
 * With tile arrays NULL it only counts.  Returns the number of listed tiles, or a
 * negative error (capacity exceeded / bad input). */
long long ora_plan_brute(int n_heads, const int32_t *ext_diag_ptr, const int32_t *ext_diag_offsets,
                         const int32_t *ext_vert_ptr, const int32_t *ext_vert_cols, int S,
                         long long capacity, int32_t *tile_ptr, int32_t *tile_key0,
                         uint64_t *tile_dmask, uint64_t *tile_cmask, uint32_t *tile_flags,
                         int32_t *stripe_cnt) {
    if (n_heads < 0 || S <= 0) return ORA_ERR_INVALID;
    const int T = ORA_TILE;
    int nqb = (S + T - 1) / T;
    uint8_t *isD = (uint8_t *)malloc((size_t)S);
    uint8_t *isC = (uint8_t *)malloc((size_t)S);
    uint8_t *need = (uint8_t *)malloc((size_t)nqb * T);
    if (!isD || !isC || !need) {
        free(isD);
        free(isC);
        free(need);
        return ORA_ERR_NOMEM;
    }
    long long n = 0;
    for (int h = 0; h < n_heads; ++h) {
        memset(isD, 0, (size_t)S);
        memset(isC, 0, (size_t)S);
        const int32_t *D = ext_diag_offsets + ext_diag_ptr[h];
        int nd = ext_diag_ptr[h + 1] - ext_diag_ptr[h];
        const int32_t *C = ext_vert_cols + ext_vert_ptr[h];
        int nc = ext_vert_ptr[h + 1] - ext_vert_ptr[h];
        for (int k = 0; k < nd; ++k) isD[D[k]] = 1;
        for (int k = 0; k < nc; ++k) isC[C[k]] = 1;
        for (int qb = 0; qb < nqb; ++qb) {
            if (tile_ptr) tile_ptr[h * nqb + qb] = (int32_t)n;
            const long lo = (long)T * qb, hi = lo + T - 1;
            int last_row = (hi < S - 1) ? (int)hi : S - 1;
            if (stripe_cnt) stripe_cnt[h * nqb + qb] = count_le(C, nc, last_row);
            /* needed keys, cell by cell over the 128 rows of the block */
            memset(need, 0, (size_t)(hi + 1));
            for (long j = 0; j <= hi; ++j)
                for (int il = 0; il < T; ++il) {
                    long r = lo + il - j;
                    if (r >= 0 && r < S && isD[r]) {
                        need[j] = 1;
                        break;
                    }
                }
            long next = 0; /* smallest allowed start of the next window */
            while (1) {
                long key0 = next;
                while (key0 <= hi && !need[key0]) ++key0;
                if (key0 > hi) break;
                next = key0 + T;
                uint64_t dm[4] = {0, 0, 0, 0}, cm[2] = {0, 0};
                for (int t = 0; t < 2 * T - 1; ++t) {
                    long r = lo - key0 + t - (T - 1);
                    if (r >= 0 && r < S && isD[r]) set_bit(dm, t);
                }
                for (int jl = 0; jl < T; ++jl) {
                    long j = key0 + jl;
                    if (j < S && isC[j]) set_bit(cm, jl);
                }
                int listed = 0;
                for (int il = 0; il < T && !listed; ++il) {
                    long i = lo + il;
                    if (i >= S) break;
                    for (int jl = 0; jl < T; ++jl) {
                        long j = key0 + jl;
                        if (j <= i && isD[i - j] && !isC[j]) {
                            listed = 1;
                            break;
                        }
                    }
                }
                if (!listed) continue;
                int full = ((long)T * (qb + 1) <= S) && popcount256(dm) == 2 * T - 1 && cm[0] == 0 &&
                           cm[1] == 0;
                if (tile_key0) {
                    if (n >= capacity) {
                        free(isD);
                        free(isC);
                        free(need);
                        return ORA_ERR_CAPACITY;
                    }
                    tile_key0[n] = (int32_t)key0;
                    memcpy(tile_dmask + 4 * n, dm, sizeof dm);
                    memcpy(tile_cmask + 2 * n, cm, sizeof cm);
                    tile_flags[n] = full ? 1u : 0u;
                }
                ++n;
            }
        }
    }
    if (tile_ptr) tile_ptr[n_heads * nqb] = (int32_t)n;
    free(isD);
    free(isC);
    free(need);
    return n;
}

/* First index k of the ascending array a[0..n) with a[k] >= x. */
static int first_ge(const int32_t *a, int n, long x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        int mid = (lo + hi) / 2;
        if (a[mid] < x) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

/* Routine 2 for one (head, query block): interval arithmetic over the offsets.
 * The diagonals r <= hi split into runs whose consecutive offsets differ by <= 128;
 * a run [ra, rb] reaches exactly the contiguous keys [max(0, lo - rb), hi - ra] from
 * the block's 128 rows, and runs further apart leave a gap of unreached keys (run0[k]
 * is the first index of the run holding D[k]).  The
 * runs, taken from the largest offset down (ascending keys), give the windows by
 * stepping 128 keys at a time from max(run start, next allowed start).  dmask / cmask
 * are range queries on the sorted lists; "listed" checks, per set dmask bit, whether
 * the diagonal's cells in valid rows reach a column outside cmask.  Appends the
 * block's tiles at out index n; returns the new n or a negative error. */
static long long interval_block(const int32_t *D, const int32_t *run0, int nd, const int32_t *C,
                                int nc, int S, int qb, long long n, long long capacity,
                                int32_t *tile_key0,
                                uint64_t *tile_dmask, uint64_t *tile_cmask, uint32_t *tile_flags) {
    const int T = ORA_TILE;
    long lo = (long)T * qb, hi = lo + T - 1;
    long hi_valid = hi < S - 1 ? hi : S - 1;
    int nrows = (int)(hi_valid - lo + 1);
    int k = first_ge(D, nd, hi + 1) - 1; /* largest offset <= hi */
    long next = 0;                          /* smallest allowed start of the next window */
    while (k >= 0) {
        int ks = run0[k];
        long a = lo - D[k] > 0 ? lo - D[k] : 0, b = hi - D[ks];
        for (long key0 = a > next ? a : next; key0 <= b; key0 += T) {
            next = key0 + T;
            long base = lo - key0 - (T - 1); /* r of dmask bit 0 */
            uint64_t dm[4] = {0, 0, 0, 0}, cm[2] = {0, 0};
            for (int q = first_ge(D, nd, base); q < nd && D[q] <= base + 2 * T - 2; ++q)
                set_bit(dm, (int)(D[q] - base));
            for (int q = first_ge(C, nc, key0); q < nc && C[q] < key0 + T; ++q)
                set_bit(cm, (int)(C[q] - key0));
            int listed = 0;
            for (int t = 0; t <= 2 * T - 2 && !listed; ++t) {
                if (!get_bit(dm, t)) continue;
                int delta = t - (T - 1); /* il - jl */
                int il_lo = delta > 0 ? delta : 0;
                int il_hi = T - 1;
                if (T - 1 + delta < il_hi) il_hi = T - 1 + delta;
                if (nrows - 1 < il_hi) il_hi = nrows - 1;
                for (int il = il_lo; il <= il_hi; ++il) {
                    if (!get_bit(cm, il - delta)) {
                        listed = 1;
                        break;
                    }
                }
            }
            if (!listed) continue;
            int full = ((long)T * (qb + 1) <= S) && popcount256(dm) == 2 * T - 1 && cm[0] == 0 &&
                       cm[1] == 0;
            if (tile_key0) {
                if (n >= capacity) return ORA_ERR_CAPACITY;
                tile_key0[n] = (int32_t)key0;
                memcpy(tile_dmask + 4 * n, dm, sizeof dm);
                memcpy(tile_cmask + 2 * n, cm, sizeof cm);
                tile_flags[n] = full ? 1u : 0u;
            }
            ++n;
        }
        k = ks - 1;
    }
    return n;
}

/* run0[k] = first index of the run of D (consecutive offsets <= 128 apart) holding D[k]. */
static void run_starts(const int32_t *D, int nd, int32_t *run0) {
    for (int k = 0; k < nd; ++k) run0[k] = (k > 0 && D[k] - D[k - 1] <= ORA_TILE) ? run0[k - 1] : k;
}

/* Routine 2 over every (head, query block); same outputs as routine 1. */
long long ora_plan_interval(int n_heads, const int32_t *ext_diag_ptr,
                            const int32_t *ext_diag_offsets, const int32_t *ext_vert_ptr,
                            const int32_t *ext_vert_cols, int S, long long capacity,
                            int32_t *tile_ptr, int32_t *tile_key0, uint64_t *tile_dmask,
                            uint64_t *tile_cmask, uint32_t *tile_flags, int32_t *stripe_cnt) {
    if (n_heads < 0 || S <= 0) return ORA_ERR_INVALID;
    const int T = ORA_TILE;
    int nqb = (S + T - 1) / T;
    int32_t *run0 = (int32_t *)malloc(sizeof(int32_t) * (size_t)(S + 1));
    if (!run0) return ORA_ERR_NOMEM;
    long long n = 0;
    for (int h = 0; h < n_heads && n >= 0; ++h) {
        const int32_t *D = ext_diag_offsets + ext_diag_ptr[h];
        int nd = ext_diag_ptr[h + 1] - ext_diag_ptr[h];
        const int32_t *C = ext_vert_cols + ext_vert_ptr[h];
        int nc = ext_vert_ptr[h + 1] - ext_vert_ptr[h];
        run_starts(D, nd, run0);
        for (int qb = 0; qb < nqb && n >= 0; ++qb) {
            if (tile_ptr) tile_ptr[h * nqb + qb] = (int32_t)n;
            long hi_i = (long)T * qb + T - 1 < S - 1 ? (long)T * qb + T - 1 : S - 1;
            if (stripe_cnt) stripe_cnt[h * nqb + qb] = count_le(C, nc, (int32_t)hi_i);
            n = interval_block(D, run0, nd, C, nc, S, qb, n, capacity, tile_key0, tile_dmask,
                               tile_cmask, tile_flags);
        }
    }
    if (tile_ptr && n >= 0) tile_ptr[n_heads * nqb] = (int32_t)n;
    free(run0);
    return n;
}

/* Routine 2 for selected blocks only (items[2a] = head, items[2a+1] = query block):
 * item_ptr[n_items+1] indexes the concatenated tiles of the items in order. */
long long ora_plan_items(int n_heads, const int32_t *ext_diag_ptr, const int32_t *ext_diag_offsets,
                         const int32_t *ext_vert_ptr, const int32_t *ext_vert_cols, int S,
                         int n_items, const int32_t *items, long long capacity, int32_t *item_ptr,
                         int32_t *tile_key0, uint64_t *tile_dmask, uint64_t *tile_cmask,
                         uint32_t *tile_flags, int32_t *stripe_cnt) {
    if (n_heads < 0 || S <= 0 || n_items < 0) return ORA_ERR_INVALID;
    const int T = ORA_TILE;
    int nqb = (S + T - 1) / T;
    int32_t *run0 = (int32_t *)malloc(sizeof(int32_t) * (size_t)(S + 1));
    if (!run0) return ORA_ERR_NOMEM;
    long long n = 0;
    for (int a = 0; a < n_items && n >= 0; ++a) {
        int h = items[2 * a], qb = items[2 * a + 1];
        if (h < 0 || h >= n_heads || qb < 0 || qb >= nqb) {
            n = ORA_ERR_INVALID;
            break;
        }
        const int32_t *D = ext_diag_offsets + ext_diag_ptr[h];
        int nd = ext_diag_ptr[h + 1] - ext_diag_ptr[h];
        const int32_t *C = ext_vert_cols + ext_vert_ptr[h];
        int nc = ext_vert_ptr[h + 1] - ext_vert_ptr[h];
        if (item_ptr) item_ptr[a] = (int32_t)n;
        long hi_i = (long)T * qb + T - 1 < S - 1 ? (long)T * qb + T - 1 : S - 1;
        if (stripe_cnt) stripe_cnt[a] = count_le(C, nc, (int32_t)hi_i);
        run_starts(D, nd, run0);
        n = interval_block(D, run0, nd, C, nc, S, qb, n, capacity, tile_key0, tile_dmask, tile_cmask,
                           tile_flags);
    }
    if (item_ptr && n >= 0) item_ptr[n_items] = (int32_t)n;
    free(run0);
    return n;
}

/* ----------------------------------------------------------------------------------
 * Attention over the extended mask: for head h (KV head g) and query row i the
 * retained key set is J_i = {i - r : r in D_h, r <= i} U {c in C_h : c <= i}; the
 * logits s_j = scale * q_i . k_j are soft-maxed over J_i only; O_i = sum_j p_j v_j,
 * LSE_i = log sum_j exp(s_j).  Empty J_i gives O_i = 0 and LSE_i = -inf.
 * -------------------------------------------------------------------------------- */

static int kv_head(int h, int Hq, int Hkv, const int32_t *kv_map) {
    return kv_map ? kv_map[h] : h / (Hq / Hkv);
}

static void attend_row(const uint16_t *q, const uint16_t *K, const uint16_t *V, int d, double scale,
                       const int32_t *J, int nJ, double *s, double *o, double *lse) {
    for (int k = 0; k < d; ++k) o[k] = 0.0;
    if (nJ == 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int a = 0; a < nJ; ++a) {
        const uint16_t *kj = K + (size_t)J[a] * d;
        double dot = 0.0;
        for (int k = 0; k < d; ++k) dot += bf16_bits_to_double(q[k]) * bf16_bits_to_double(kj[k]);
        s[a] = scale * dot;
        if (s[a] > m) m = s[a];
    }
    double l = 0.0;
    for (int a = 0; a < nJ; ++a) {
        double p = exp(s[a] - m);
        s[a] = p;
        l += p;
    }
    for (int a = 0; a < nJ; ++a) {
        const uint16_t *vj = V + (size_t)J[a] * d;
        for (int k = 0; k < d; ++k) o[k] += s[a] * bf16_bits_to_double(vj[k]);
    }
    for (int k = 0; k < d; ++k) o[k] /= l;
    *lse = m + log(l);
}

/* List-driven attention for a chosen set of query rows (the same rows in every head).
 * Q [Hq][S][d], K/V [Hkv][S][d] bf16 bits; O [Hq][n_rows][d], LSE [Hq][n_rows]. */
int ora_attn_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int Hq, int Hkv, int S,
                  int d, const int32_t *ext_diag_ptr, const int32_t *ext_diag_offsets,
                  const int32_t *ext_vert_ptr, const int32_t *ext_vert_cols,
                  const int32_t *kv_map, double scale, int n_rows, const int32_t *rows, double *O,
                  double *LSE) {
    if (!Q || !K || !V || Hq <= 0 || Hkv <= 0 || S <= 0 || d <= 0) return ORA_ERR_INVALID;
    if (!kv_map && Hq % Hkv != 0) return ORA_ERR_INVALID;
    for (int a = 0; a < n_rows; ++a)
        if (rows[a] < 0 || rows[a] >= S) return ORA_ERR_INVALID;
    int err = ORA_OK;
#pragma omp parallel
    {
        uint8_t *mark = (uint8_t *)calloc((size_t)S, 1);
        int32_t *J = (int32_t *)malloc(sizeof(int32_t) * (size_t)S);
        double *s = (double *)malloc(sizeof(double) * (size_t)S);
        if (!mark || !J || !s) err = ORA_ERR_NOMEM;
#pragma omp for schedule(dynamic, 4) collapse(2)
        for (int h = 0; h < Hq; ++h) {
            for (int a = 0; a < n_rows; ++a) {
                if (!mark || !J || !s) continue;
                int g = kv_head(h, Hq, Hkv, kv_map);
                const int32_t *D = ext_diag_offsets + ext_diag_ptr[h];
                int nd = ext_diag_ptr[h + 1] - ext_diag_ptr[h];
                const int32_t *C = ext_vert_cols + ext_vert_ptr[h];
                int nc = ext_vert_ptr[h + 1] - ext_vert_ptr[h];
                long i = rows[a];
                int nJ = 0;
                for (int k = 0; k < nd; ++k) {
                    if (D[k] > i) continue;
                    int32_t j = (int32_t)(i - D[k]);
                    if (!mark[j]) {
                        mark[j] = 1;
                        J[nJ++] = j;
                    }
                }
                for (int k = 0; k < nc; ++k) {
                    if (C[k] > i) continue;
                    if (!mark[C[k]]) {
                        mark[C[k]] = 1;
                        J[nJ++] = C[k];
                    }
                }
                for (int b = 0; b < nJ; ++b) mark[J[b]] = 0;
                attend_row(Q + ((size_t)h * S + i) * d, K + (size_t)g * S * d, V + (size_t)g * S * d,
                           d, scale, J, nJ, s, O + ((size_t)h * n_rows + a) * d,
                           LSE + (size_t)h * n_rows + a);
            }
        }
        free(mark);
        free(J);
        free(s);
    }
    return err;
}

/* Dense-mask attention (small S): materialises the S x S boolean extended mask as the
 * union of every kept pattern's cells, then soft-maxes each row over its set cells in
 * ascending key order.  With `block` (uint8 [Hq][Lb][Lb], may be NULL) the first
 * Lb x Lb cells of head h are replaced by block[h] (j <= i only): the Case-2 reading
 * of the extended mask.  O [Hq][S][d], LSE [Hq][S]. */
static int attn_dense_impl(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int Hq, int Hkv, int S,
                           int d, const int32_t *ext_diag_ptr, const int32_t *ext_diag_offsets,
                           const int32_t *ext_vert_ptr, const int32_t *ext_vert_cols,
                           const int32_t *kv_map, double scale, const uint8_t *block, int Lb, double *O,
                           double *LSE) {
    if (!Q || !K || !V || Hq <= 0 || Hkv <= 0 || S <= 0 || S > 8192 || d <= 0)
        return ORA_ERR_INVALID;
    if (!kv_map && Hq % Hkv != 0) return ORA_ERR_INVALID;
    if (block && Lb <= 0) return ORA_ERR_INVALID;
    uint8_t *Mt = (uint8_t *)malloc((size_t)S * S);
    if (!Mt) return ORA_ERR_NOMEM;
    int err = ORA_OK;
    for (int h = 0; h < Hq && err == ORA_OK; ++h) {
        memset(Mt, 0, (size_t)S * S);
        const int32_t *D = ext_diag_offsets + ext_diag_ptr[h];
        int nd = ext_diag_ptr[h + 1] - ext_diag_ptr[h];
        const int32_t *C = ext_vert_cols + ext_vert_ptr[h];
        int nc = ext_vert_ptr[h + 1] - ext_vert_ptr[h];
        for (int k = 0; k < nd; ++k)
            for (long i = D[k]; i < S; ++i) Mt[(size_t)i * S + (i - D[k])] = 1;
        for (int k = 0; k < nc; ++k)
            for (long i = C[k]; i < S; ++i) Mt[(size_t)i * S + C[k]] = 1;
        if (block) {
            const uint8_t *Bh = block + (size_t)h * Lb * Lb;
            int lim = Lb < S ? Lb : S;
            for (int i = 0; i < lim; ++i)
                for (int j = 0; j <= i; ++j) Mt[(size_t)i * S + j] = Bh[(size_t)i * Lb + j] ? 1 : 0;
        }
        int g = kv_head(h, Hq, Hkv, kv_map);
#pragma omp parallel
        {
            int32_t *J = (int32_t *)malloc(sizeof(int32_t) * (size_t)S);
            double *s = (double *)malloc(sizeof(double) * (size_t)S);
            if (!J || !s) err = ORA_ERR_NOMEM;
#pragma omp for schedule(dynamic, 8)
            for (int i = 0; i < S; ++i) {
                if (!J || !s) continue;
                int nJ = 0;
                for (int j = 0; j <= i; ++j)
                    if (Mt[(size_t)i * S + j]) J[nJ++] = j;
                attend_row(Q + ((size_t)h * S + i) * d, K + (size_t)g * S * d, V + (size_t)g * S * d,
                           d, scale, J, nJ, s, O + ((size_t)h * S + i) * d, LSE + (size_t)h * S + i);
            }
            free(J);
            free(s);
        }
    }
    free(Mt);
    return err;
}

int ora_attn_dense(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int Hq, int Hkv, int S,
                   int d, const int32_t *ext_diag_ptr, const int32_t *ext_diag_offsets,
                   const int32_t *ext_vert_ptr, const int32_t *ext_vert_cols,
                   const int32_t *kv_map, double scale, double *O, double *LSE) {
    return attn_dense_impl(Q, K, V, Hq, Hkv, S, d, ext_diag_ptr, ext_diag_offsets, ext_vert_ptr,
                           ext_vert_cols, kv_map, scale, NULL, 0, O, LSE);
}

/* Case-2 reading of the extended mask (DAM review page, Referee Report major comment 2:
 * the patterns are pasted beyond the first L tokens): the captured L x L true mask of
 * each head kept verbatim in the first L x L block, the union of the kept patterns
 * everywhere else.  true_masks uint8 [Hq][L][L] (entries j > i ignored). */
int ora_attn_dense_case2(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int Hq, int Hkv, int S,
                         int d, const int32_t *ext_diag_ptr, const int32_t *ext_diag_offsets,
                         const int32_t *ext_vert_ptr, const int32_t *ext_vert_cols,
                         const int32_t *kv_map, double scale, const uint8_t *true_masks, int L, double *O,
                         double *LSE) {
    if (!true_masks) return ORA_ERR_INVALID;
    return attn_dense_impl(Q, K, V, Hq, Hkv, S, d, ext_diag_ptr, ext_diag_offsets, ext_vert_ptr,
                           ext_vert_cols, kv_map, scale, true_masks, L, O, LSE);
}

/* Number of retained (i, j) pairs of each head over the S x S extended mask, counted
 * from the list form: |J_i| summed over rows (for the effective-FLOP metric). */
int ora_nnz(int n_heads, const int32_t *ext_diag_ptr, const int32_t *ext_diag_offsets,
            const int32_t *ext_vert_ptr, const int32_t *ext_vert_cols, int S, long long *nnz) {
    for (int h = 0; h < n_heads; ++h) {
        const int32_t *D = ext_diag_offsets + ext_diag_ptr[h];
        int nd = ext_diag_ptr[h + 1] - ext_diag_ptr[h];
        const int32_t *C = ext_vert_cols + ext_vert_ptr[h];
        int nc = ext_vert_ptr[h + 1] - ext_vert_ptr[h];
        long long total = 0;
        /* each diagonal r contributes S - r cells; each column c contributes S - c cells;
         * a cell on both (i - c in D_h) is counted once */
        for (int k = 0; k < nd; ++k) total += (long long)S - D[k];
        for (int k = 0; k < nc; ++k) {
            long long own = (long long)S - C[k];
            long long shared = 0;
            for (int q = 0; q < nd; ++q)
                if ((long long)C[k] + D[q] < S) ++shared;
            total += own - shared;
        }
        nnz[h] = total;
    }
    return ORA_OK;
}

/* Averaged attention maps, the input of stage one ("What carries the argument":
 * attention maps averaged over a calibration corpus at capture length L).  For map m,
 * sample b and row i: the causal logits s_j = scale * <q_i, k_j> (j <= i), their
 * softmax p_j = exp(s_j - max) / sum_j' exp(s_j' - max), and
 *   maps[m][i][j] = (1/B) sum_b p_j  (j <= i),   0 above the diagonal.
 * Q, K bf16 bits [n_maps][B][L][d]; maps [n_maps][L][L] in fp64. */
int ora_attn_maps(const uint16_t *Q, const uint16_t *K, int n_maps, int B, int L, int d, double scale,
                  double *maps) {
    if (!Q || !K || !maps || n_maps <= 0 || B <= 0 || L <= 0 || d <= 0) return ORA_ERR_INVALID;
    int err = ORA_OK;
    memset(maps, 0, sizeof(double) * (size_t)n_maps * L * L);
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)L);
        if (!s) err = ORA_ERR_NOMEM;
#pragma omp for schedule(dynamic, 1)
        for (int m = 0; m < n_maps; ++m) {
            if (!s) continue;
            for (int b = 0; b < B; ++b) {
                const uint16_t *q = Q + ((size_t)m * B + b) * L * d;
                const uint16_t *k = K + ((size_t)m * B + b) * L * d;
                for (int i = 0; i < L; ++i) {
                    double mx = -INFINITY;
                    for (int j = 0; j <= i; ++j) {
                        double dot = 0.0;
                        for (int c = 0; c < d; ++c)
                            dot += bf16_bits_to_double(q[(size_t)i * d + c]) * bf16_bits_to_double(k[(size_t)j * d + c]);
                        s[j] = scale * dot;
                        if (s[j] > mx) mx = s[j];
                    }
                    double sum = 0.0;
                    for (int j = 0; j <= i; ++j) {
                        s[j] = exp(s[j] - mx);
                        sum += s[j];
                    }
                    double *row = maps + ((size_t)m * L + i) * L;
                    for (int j = 0; j <= i; ++j) row[j] += s[j] / sum / B;
                }
            }
        }
        free(s);
    }
    return err;
}
