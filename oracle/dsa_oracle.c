/*
 * fp64 CPU oracle for 3D Deformable Slide Attention (3D-DSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file: only the
 * tests, the smoke check and the benchmark's CPU-baseline leg use it.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (plain definition, no blocking, fusion or reordering):
 *
 *   Operator: "3D Deformable Slide Attention (3D-DSA), a motion-adaptive local attention
 *   operator" whose cost is linear in the sequence length ("MegaSlide-DiT: Memory-Centric
 *   Adaptation and Deformable Local Attention for Efficient Video Diffusion", abstract),
 *   in the tile-granular local 3D window form of "Fast Video Generation with Sliding Tile
 *   Attention" (abstract: attending over a local spatial-temporal region).
 *
 *   Concrete form used here (the pages give only the outline above):
 *     - the token grid T x H x W is cut into tiles tt x th x tw; tile grid G = (T/tt, H/th, W/tw);
 *     - per axis the window length is w' = min(w, G) tiles;
 *     - query tile i with integer offset o (tile units) gets the window start
 *           s = clamp(i + o - floor(w'/2), 0, G - w')
 *       per axis, and its key set K(i) is every token of the tiles j with s <= j < s + w'
 *       on all three axes;
 *     - for query token n in tile i:  s_nm = scale * <q_n, k_m>,  m in K(i);
 *           lse_n = ln sum_m exp(s_nm),   o_n = sum_m exp(s_nm - lse_n) v_m;
 *     - backward of L = sum_n <o_n, dO_n>:
 *           P_nm = exp(s_nm - lse_n),  dP_nm = <dO_n, v_m>,
 *           dS_nm = P_nm (dP_nm - sum_m' P_nm' dP_nm'),
 *           dq_n = scale sum_m dS_nm k_m,  dk_m = scale sum_n dS_nm q_n,  dv_m = sum_n P_nm dO_n,
 *       where the sums for dk_m and dv_m run over every query token n whose key set holds m.
 *
 * Inputs and every arithmetic step are double (bf16 and fp32 inputs widen to it exactly).  Token tensors are [B, heads, T, H, W, d] contiguous; offsets are
 * int32 [nTiles, 3] (dt, dh, dw) in tile-raster order (t outer, w inner).
 *
 *   Key-tile-list form (block-sparse attention, the generalisation of the box to an
 *   arbitrary per-query-tile list of key tiles, as in the MOD-DiT page's Method section,
 *   Stage 2, online block masking):
 *   K(i) is every token of the tiles listed for i in a CSR (row_ptr, list); a tile listed
 *   twice counts twice; an empty list gives o = 0 and lse = -inf.  Functions *_list.
 *
 *   Block attention mass (oracle_block_map_list): the mean over a query tile's tokens of
 *   the probability mass each listed key tile receives.
 *
 *   Text prefix (oracle_fwd_prefix; the MOD-DiT page, "Token-Type-Aware Masking"): a video
 *   query attends to its window and to every text token in one softmax.
 *
 * Parity pins (tests, CPU only): a window covering the grid equals dense attention; a
 * 1x1x1 window equals block-diagonal attention; softmax rows sum to one; brute-force
 * membership by nearest window centre; backward against central finite differences;
 * lists: multiset-weighted dense attention and its autograd backward, doubled lists
 * (same o, lse + ln 2), lists of the window plan equal the window form; block map: blocked
 * dense probabilities; text prefix: masked dense attention over the unified sequence.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t B, heads, d;
    int32_t T, H, W;
    int32_t tt, th, tw;
    int32_t wt, wh, ww;
    double scale;
} oracle_problem;

static int32_t min_i(int32_t a, int32_t b) { return a < b ? a : b; }

static int32_t clamp_i(int32_t x, int32_t lo, int32_t hi) {
    if (x < lo) return lo;
    if (x > hi) return hi;
    return x;
}

/* Window start along one axis: centre = tile index + offset, start = centre - floor(w'/2),
 * then moved so that [start, start + w') lies inside [0, G). */
static int32_t axis_start(int32_t tile_index, int32_t offset, int32_t w_eff, int32_t G) {
    return clamp_i(tile_index + offset - w_eff / 2, 0, G - w_eff);
}

typedef struct {
    int32_t G[3];   /* tile grid (Gt, Gh, Gw) */
    int32_t w[3];   /* effective window (w't, w'h, w'w) */
    int32_t n_tiles, n_window_tiles, tile_tokens, n_tokens;
} geometry;

static int make_geometry(const oracle_problem* p, geometry* g) {
    if (p->tt <= 0 || p->th <= 0 || p->tw <= 0) return 1;
    if (p->T % p->tt || p->H % p->th || p->W % p->tw) return 1;
    if (p->wt <= 0 || p->wh <= 0 || p->ww <= 0) return 1;
    g->G[0] = p->T / p->tt;
    g->G[1] = p->H / p->th;
    g->G[2] = p->W / p->tw;
    g->w[0] = min_i(p->wt, g->G[0]);
    g->w[1] = min_i(p->wh, g->G[1]);
    g->w[2] = min_i(p->ww, g->G[2]);
    g->n_tiles = g->G[0] * g->G[1] * g->G[2];
    g->n_window_tiles = g->w[0] * g->w[1] * g->w[2];
    g->tile_tokens = p->tt * p->th * p->tw;
    g->n_tokens = p->T * p->H * p->W;
    return 0;
}

static void tile_coords(const geometry* g, int32_t tile, int32_t c[3]) {
    c[2] = tile % g->G[2];
    c[1] = (tile / g->G[2]) % g->G[1];
    c[0] = tile / (g->G[2] * g->G[1]);
}

static void window_starts(const geometry* g, const int32_t* offsets, int32_t tile, int32_t s[3]) {
    int32_t c[3];
    tile_coords(g, tile, c);
    for (int a = 0; a < 3; ++a) s[a] = axis_start(c[a], offsets[3 * tile + a], g->w[a], g->G[a]);
}

static int window_holds(const geometry* g, const int32_t s[3], int32_t key_tile) {
    int32_t c[3];
    tile_coords(g, key_tile, c);
    for (int a = 0; a < 3; ++a)
        if (c[a] < s[a] || c[a] >= s[a] + g->w[a]) return 0;
    return 1;
}

/* Position of a key tile in the raster order (t outer, w inner) of a window box that holds it. */
static int64_t window_position(const geometry* g, const int32_t s[3], int32_t key_tile) {
    int32_t c[3];
    tile_coords(g, key_tile, c);
    return ((int64_t)(c[0] - s[0]) * g->w[1] + (c[1] - s[1])) * g->w[2] + (c[2] - s[2]);
}

/* Token index (within one (b, head) slice) of the r-th token of a tile, tokens of a tile
 * taken in raster order (t outer, w inner). */
static int64_t tile_token(const oracle_problem* p, const geometry* g, int32_t tile, int32_t r) {
    int32_t c[3];
    tile_coords(g, tile, c);
    int32_t lw = r % p->tw, lh = (r / p->tw) % p->th, lt = r / (p->tw * p->th);
    int64_t t = (int64_t)c[0] * p->tt + lt, h = (int64_t)c[1] * p->th + lh, w = (int64_t)c[2] * p->tw + lw;
    return (t * p->H + h) * p->W + w;
}

/* Token indices of K(i), key tiles in raster order of the window box, tokens of each
 * tile in raster order.  keys must hold n_window_tiles * tile_tokens entries. */
static void key_set(const oracle_problem* p, const geometry* g, const int32_t* offsets, int32_t tile,
                    int64_t* keys) {
    int32_t s[3];
    window_starts(g, offsets, tile, s);
    int64_t n = 0;
    for (int32_t a = s[0]; a < s[0] + g->w[0]; ++a)
        for (int32_t b = s[1]; b < s[1] + g->w[1]; ++b)
            for (int32_t c = s[2]; c < s[2] + g->w[2]; ++c) {
                int32_t kt = (a * g->G[1] + b) * g->G[2] + c;
                for (int32_t r = 0; r < g->tile_tokens; ++r) keys[n++] = tile_token(p, g, kt, r);
            }
}

static double dot(const double* x, const double* y, int32_t d) {
    double acc = 0.0;
    for (int32_t c = 0; c < d; ++c) acc += x[c] * y[c];
    return acc;
}

/* Scores of query token n over its key set, its log-sum-exp (max subtracted), and the
 * softmax row P (written over the scores). */
static double softmax_row(const oracle_problem* p, const double* qrow, const double* kbase, const int64_t* keys,
                          int64_t nk, double* P) {
    double mx = -INFINITY;
    for (int64_t m = 0; m < nk; ++m) {
        P[m] = p->scale * dot(qrow, kbase + keys[m] * p->d, p->d);
        if (P[m] > mx) mx = P[m];
    }
    double sum = 0.0;
    for (int64_t m = 0; m < nk; ++m) sum += exp(P[m] - mx);
    double lse = mx + log(sum);
    for (int64_t m = 0; m < nk; ++m) P[m] = exp(P[m] - lse);
    return lse;
}

/* ---------------------------------------------------------------------------------- */

/* Window plan: starts[nTiles,3], kv_tiles[nTiles, Wt] (key tiles of each window in
 * ascending linear index), and the inverse map as CSR: row j lists, ascending, the query
 * tiles whose window holds key tile j.  row_ptr / q_tiles may be NULL.  Returns 0 on
 * success, 1 on an invalid shape. */
int oracle_plan(int32_t Gt, int32_t Gh, int32_t Gw, int32_t wt, int32_t wh, int32_t ww, const int32_t* offsets,
                int32_t* starts, int32_t* kv_tiles, int32_t* row_ptr, int32_t* q_tiles) {
    if (Gt <= 0 || Gh <= 0 || Gw <= 0 || wt <= 0 || wh <= 0 || ww <= 0) return 1;
    geometry g;
    g.G[0] = Gt; g.G[1] = Gh; g.G[2] = Gw;
    g.w[0] = min_i(wt, Gt); g.w[1] = min_i(wh, Gh); g.w[2] = min_i(ww, Gw);
    g.n_tiles = Gt * Gh * Gw;
    g.n_window_tiles = g.w[0] * g.w[1] * g.w[2];
    for (int32_t i = 0; i < g.n_tiles; ++i) {
        int32_t s[3];
        window_starts(&g, offsets, i, s);
        for (int a = 0; a < 3; ++a) starts[3 * i + a] = s[a];
        int32_t n = 0;
        for (int32_t a = s[0]; a < s[0] + g.w[0]; ++a)
            for (int32_t b = s[1]; b < s[1] + g.w[1]; ++b)
                for (int32_t c = s[2]; c < s[2] + g.w[2]; ++c)
                    kv_tiles[(int64_t)i * g.n_window_tiles + n++] = (a * Gh + b) * Gw + c;
    }
    if (row_ptr && q_tiles) {
        int32_t n = 0;
        for (int32_t j = 0; j < g.n_tiles; ++j) {
            row_ptr[j] = n;
            for (int32_t i = 0; i < g.n_tiles; ++i) {
                int32_t s[3];
                window_starts(&g, offsets, i, s);
                if (window_holds(&g, s, j)) q_tiles[n++] = i;
            }
        }
        row_ptr[g.n_tiles] = n;
    }
    return 0;
}

/* Forward on selected (b*heads + head, query tile) pairs.
 * out: [n_sel][tile_tokens][d], lse: [n_sel][tile_tokens]; rows of a selection are the
 * tokens of its query tile in raster order. */
int oracle_fwd(const oracle_problem* p, const double* q, const double* k, const double* v, const int32_t* offsets,
               int32_t n_sel, const int32_t* sel_bh, const int32_t* sel_tile, double* out, double* lse) {
    geometry g;
    if (make_geometry(p, &g)) return 1;
    const int64_t nk = (int64_t)g.n_window_tiles * g.tile_tokens;
    const int64_t slice = (int64_t)g.n_tokens * p->d;
    int status = 0;
#pragma omp parallel
    {
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * nk);
        double* P = (double*)malloc(sizeof(double) * nk);
        if (!keys || !P) {
#pragma omp atomic write
            status = 2;
        }
#pragma omp for schedule(dynamic)
        for (int64_t job = 0; job < (int64_t)n_sel * g.tile_tokens; ++job) {
            if (!keys || !P) continue;
            int32_t s = (int32_t)(job / g.tile_tokens), r = (int32_t)(job % g.tile_tokens);
            const double* qb = q + sel_bh[s] * slice;
            const double* kb = k + sel_bh[s] * slice;
            const double* vb = v + sel_bh[s] * slice;
            key_set(p, &g, offsets, sel_tile[s], keys);
            int64_t n = tile_token(p, &g, sel_tile[s], r);
            double l = softmax_row(p, qb + n * p->d, kb, keys, nk, P);
            double* o = out + ((int64_t)s * g.tile_tokens + r) * p->d;
            for (int32_t c = 0; c < p->d; ++c) o[c] = 0.0;
            for (int64_t m = 0; m < nk; ++m) {
                const double* vm = vb + keys[m] * p->d;
                for (int32_t c = 0; c < p->d; ++c) o[c] += P[m] * vm[c];
            }
            lse[(int64_t)s * g.tile_tokens + r] = l;
        }
        free(keys);
        free(P);
    }
    return status;
}

/* Backward for dq on selected (bh, query tile) pairs.  dq: [n_sel][tile_tokens][d]. */
int oracle_bwd_dq(const oracle_problem* p, const double* q, const double* k, const double* v, const double* dout,
                  const int32_t* offsets, int32_t n_sel, const int32_t* sel_bh, const int32_t* sel_tile, double* dq) {
    geometry g;
    if (make_geometry(p, &g)) return 1;
    const int64_t nk = (int64_t)g.n_window_tiles * g.tile_tokens;
    const int64_t slice = (int64_t)g.n_tokens * p->d;
    int status = 0;
#pragma omp parallel
    {
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * nk);
        double* P = (double*)malloc(sizeof(double) * nk);
        double* dP = (double*)malloc(sizeof(double) * nk);
        if (!keys || !P || !dP) {
#pragma omp atomic write
            status = 2;
        }
#pragma omp for schedule(dynamic)
        for (int64_t job = 0; job < (int64_t)n_sel * g.tile_tokens; ++job) {
            if (!keys || !P || !dP) continue;
            int32_t s = (int32_t)(job / g.tile_tokens), r = (int32_t)(job % g.tile_tokens);
            const double* qb = q + sel_bh[s] * slice;
            const double* kb = k + sel_bh[s] * slice;
            const double* vb = v + sel_bh[s] * slice;
            const double* dob = dout + sel_bh[s] * slice;
            key_set(p, &g, offsets, sel_tile[s], keys);
            int64_t n = tile_token(p, &g, sel_tile[s], r);
            softmax_row(p, qb + n * p->d, kb, keys, nk, P);
            double D = 0.0;
            for (int64_t m = 0; m < nk; ++m) {
                dP[m] = dot(dob + n * p->d, vb + keys[m] * p->d, p->d);
                D += P[m] * dP[m];
            }
            double* o = dq + ((int64_t)s * g.tile_tokens + r) * p->d;
            for (int32_t c = 0; c < p->d; ++c) o[c] = 0.0;
            for (int64_t m = 0; m < nk; ++m) {
                double dS = P[m] * (dP[m] - D);
                const double* km = kb + keys[m] * p->d;
                for (int32_t c = 0; c < p->d; ++c) o[c] += p->scale * dS * km[c];
            }
        }
        free(keys);
        free(P);
        free(dP);
    }
    return status;
}

/* Backward for dk and dv on selected (bh, key tile) pairs.  For each selected key tile j,
 * every query token whose window holds j contributes.  dk, dv: [n_sel][tile_tokens][d],
 * rows in the key tile's raster order. */
int oracle_bwd_dkdv(const oracle_problem* p, const double* q, const double* k, const double* v, const double* dout,
                    const int32_t* offsets, int32_t n_sel, const int32_t* sel_bh, const int32_t* sel_tile,
                    double* dk, double* dv) {
    geometry g;
    if (make_geometry(p, &g)) return 1;
    const int64_t nk = (int64_t)g.n_window_tiles * g.tile_tokens;
    const int64_t slice = (int64_t)g.n_tokens * p->d;
    const int64_t tile_elems = (int64_t)g.tile_tokens * p->d;
    int32_t* q_list = (int32_t*)malloc(sizeof(int32_t) * g.n_tiles);
    if (!q_list) return 2;
    int status = 0;
    memset(dk, 0, sizeof(double) * n_sel * tile_elems);
    memset(dv, 0, sizeof(double) * n_sel * tile_elems);
    for (int32_t s = 0; s < n_sel; ++s) {
        const int32_t j = sel_tile[s];
        int32_t nq = 0;
        for (int32_t i = 0; i < g.n_tiles; ++i) {
            int32_t st[3];
            window_starts(&g, offsets, i, st);
            if (window_holds(&g, st, j)) q_list[nq++] = i;
        }
        const double* qb = q + sel_bh[s] * slice;
        const double* kb = k + sel_bh[s] * slice;
        const double* vb = v + sel_bh[s] * slice;
        const double* dob = dout + sel_bh[s] * slice;
        double* dks = dk + s * tile_elems;
        double* dvs = dv + s * tile_elems;
#pragma omp parallel
        {
            int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * nk);
            double* P = (double*)malloc(sizeof(double) * nk);
            double* dP = (double*)malloc(sizeof(double) * nk);
            double* dk_local = (double*)calloc(tile_elems, sizeof(double));
            double* dv_local = (double*)calloc(tile_elems, sizeof(double));
            int ok = keys && P && dP && dk_local && dv_local;
            if (!ok) {
#pragma omp atomic write
                status = 2;
            }
#pragma omp for schedule(dynamic)
            for (int64_t job = 0; job < (int64_t)nq * g.tile_tokens; ++job) {
                if (!ok) continue;
                int32_t i = q_list[job / g.tile_tokens], r = (int32_t)(job % g.tile_tokens);
                key_set(p, &g, offsets, i, keys);
                int64_t n = tile_token(p, &g, i, r);
                softmax_row(p, qb + n * p->d, kb, keys, nk, P);
                double D = 0.0;
                for (int64_t m = 0; m < nk; ++m) {
                    dP[m] = dot(dob + n * p->d, vb + keys[m] * p->d, p->d);
                    D += P[m] * dP[m];
                }
                /* key tile j sits at position pos of the window's tile list, so its r-th
                 * token is entry pos * tile_tokens + r of the key set */
                int32_t st[3];
                window_starts(&g, offsets, i, st);
                int64_t pos = window_position(&g, st, j);
                for (int32_t rk = 0; rk < g.tile_tokens; ++rk) {
                    int64_t m = pos * g.tile_tokens + rk;
                    double dS = P[m] * (dP[m] - D);
                    for (int32_t c = 0; c < p->d; ++c) {
                        dk_local[(int64_t)rk * p->d + c] += p->scale * dS * qb[n * p->d + c];
                        dv_local[(int64_t)rk * p->d + c] += P[m] * dob[n * p->d + c];
                    }
                }
            }
            if (ok) {
#pragma omp critical
                for (int64_t e = 0; e < tile_elems; ++e) {
                    dks[e] += dk_local[e];
                    dvs[e] += dv_local[e];
                }
            }
            free(keys);
            free(P);
            free(dP);
            free(dk_local);
            free(dv_local);
        }
    }
    free(q_list);
    return status;
}

/* ---------------------------------------------------------------------------------- */
/* Key-tile lists (the block-sparse form: a per-query-tile list of key tiles in place of
 * the window box).  Query tile i attends to every token of the key tiles
 * list[row_ptr[i]] .. list[row_ptr[i+1] - 1], in list order, tokens of a tile in raster
 * order.  A tile listed twice counts twice (the softmax runs over the multiset).  An empty
 * list gives o = 0 and lse = -inf (the log of an empty sum).  Returns 1 for a list that is
 * not a CSR over valid tiles (row_ptr[0] = 0, non-decreasing, entries in [0, nTiles)). */

static int check_lists(const geometry* g, const int32_t* row_ptr, const int32_t* list) {
    if (row_ptr[0] != 0) return 1;
    for (int32_t i = 0; i < g->n_tiles; ++i) {
        if (row_ptr[i + 1] < row_ptr[i]) return 1;
        for (int32_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e)
            if (list[e] < 0 || list[e] >= g->n_tiles) return 1;
    }
    return 0;
}

static int64_t longest_list(const geometry* g, const int32_t* row_ptr) {
    int64_t m = 0;
    for (int32_t i = 0; i < g->n_tiles; ++i)
        if (row_ptr[i + 1] - row_ptr[i] > m) m = row_ptr[i + 1] - row_ptr[i];
    return m;
}

static int64_t list_key_set(const oracle_problem* p, const geometry* g, const int32_t* row_ptr, const int32_t* list,
                            int32_t tile, int64_t* keys) {
    int64_t n = 0;
    for (int32_t e = row_ptr[tile]; e < row_ptr[tile + 1]; ++e)
        for (int32_t r = 0; r < g->tile_tokens; ++r) keys[n++] = tile_token(p, g, list[e], r);
    return n;
}

/* Forward on selected (bh, query tile) pairs over key-tile lists; layouts as oracle_fwd. */
int oracle_fwd_list(const oracle_problem* p, const double* q, const double* k, const double* v,
                    const int32_t* row_ptr, const int32_t* list, int32_t n_sel, const int32_t* sel_bh,
                    const int32_t* sel_tile, double* out, double* lse) {
    geometry g;
    if (make_geometry(p, &g) || check_lists(&g, row_ptr, list)) return 1;
    const int64_t nk_max = longest_list(&g, row_ptr) * g.tile_tokens + 1;
    const int64_t slice = (int64_t)g.n_tokens * p->d;
    int status = 0;
#pragma omp parallel
    {
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * nk_max);
        double* P = (double*)malloc(sizeof(double) * nk_max);
        if (!keys || !P) {
#pragma omp atomic write
            status = 2;
        }
#pragma omp for schedule(dynamic)
        for (int64_t job = 0; job < (int64_t)n_sel * g.tile_tokens; ++job) {
            if (!keys || !P) continue;
            int32_t s = (int32_t)(job / g.tile_tokens), r = (int32_t)(job % g.tile_tokens);
            const double* qb = q + sel_bh[s] * slice;
            const double* kb = k + sel_bh[s] * slice;
            const double* vb = v + sel_bh[s] * slice;
            int64_t nk = list_key_set(p, &g, row_ptr, list, sel_tile[s], keys);
            int64_t n = tile_token(p, &g, sel_tile[s], r);
            double* o = out + ((int64_t)s * g.tile_tokens + r) * p->d;
            for (int32_t c = 0; c < p->d; ++c) o[c] = 0.0;
            if (nk == 0) {
                lse[(int64_t)s * g.tile_tokens + r] = -INFINITY;
                continue;
            }
            double l = softmax_row(p, qb + n * p->d, kb, keys, nk, P);
            for (int64_t m = 0; m < nk; ++m) {
                const double* vm = vb + keys[m] * p->d;
                for (int32_t c = 0; c < p->d; ++c) o[c] += P[m] * vm[c];
            }
            lse[(int64_t)s * g.tile_tokens + r] = l;
        }
        free(keys);
        free(P);
    }
    return status;
}

/* dq on selected (bh, query tile) pairs over key-tile lists; zero for an empty list. */
int oracle_bwd_dq_list(const oracle_problem* p, const double* q, const double* k, const double* v, const double* dout,
                       const int32_t* row_ptr, const int32_t* list, int32_t n_sel, const int32_t* sel_bh,
                       const int32_t* sel_tile, double* dq) {
    geometry g;
    if (make_geometry(p, &g) || check_lists(&g, row_ptr, list)) return 1;
    const int64_t nk_max = longest_list(&g, row_ptr) * g.tile_tokens + 1;
    const int64_t slice = (int64_t)g.n_tokens * p->d;
    int status = 0;
#pragma omp parallel
    {
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * nk_max);
        double* P = (double*)malloc(sizeof(double) * nk_max);
        double* dP = (double*)malloc(sizeof(double) * nk_max);
        if (!keys || !P || !dP) {
#pragma omp atomic write
            status = 2;
        }
#pragma omp for schedule(dynamic)
        for (int64_t job = 0; job < (int64_t)n_sel * g.tile_tokens; ++job) {
            if (!keys || !P || !dP) continue;
            int32_t s = (int32_t)(job / g.tile_tokens), r = (int32_t)(job % g.tile_tokens);
            const double* qb = q + sel_bh[s] * slice;
            const double* kb = k + sel_bh[s] * slice;
            const double* vb = v + sel_bh[s] * slice;
            const double* dob = dout + sel_bh[s] * slice;
            int64_t nk = list_key_set(p, &g, row_ptr, list, sel_tile[s], keys);
            int64_t n = tile_token(p, &g, sel_tile[s], r);
            double* o = dq + ((int64_t)s * g.tile_tokens + r) * p->d;
            for (int32_t c = 0; c < p->d; ++c) o[c] = 0.0;
            if (nk == 0) continue;
            softmax_row(p, qb + n * p->d, kb, keys, nk, P);
            double D = 0.0;
            for (int64_t m = 0; m < nk; ++m) {
                dP[m] = dot(dob + n * p->d, vb + keys[m] * p->d, p->d);
                D += P[m] * dP[m];
            }
            for (int64_t m = 0; m < nk; ++m) {
                double dS = P[m] * (dP[m] - D);
                const double* km = kb + keys[m] * p->d;
                for (int32_t c = 0; c < p->d; ++c) o[c] += p->scale * dS * km[c];
            }
        }
        free(keys);
        free(P);
        free(dP);
    }
    return status;
}

/* dk, dv on selected (bh, key tile) pairs over key-tile lists: every occurrence of key
 * tile j in the list of query tile i contributes for every query token of i. */
int oracle_bwd_dkdv_list(const oracle_problem* p, const double* q, const double* k, const double* v,
                         const double* dout, const int32_t* row_ptr, const int32_t* list, int32_t n_sel,
                         const int32_t* sel_bh, const int32_t* sel_tile, double* dk, double* dv) {
    geometry g;
    if (make_geometry(p, &g) || check_lists(&g, row_ptr, list)) return 1;
    const int64_t nk_max = longest_list(&g, row_ptr) * g.tile_tokens + 1;
    const int64_t slice = (int64_t)g.n_tokens * p->d;
    const int64_t tile_elems = (int64_t)g.tile_tokens * p->d;
    int32_t* q_list = (int32_t*)malloc(sizeof(int32_t) * (g.n_tiles + 1));
    if (!q_list) return 2;
    int status = 0;
    memset(dk, 0, sizeof(double) * n_sel * tile_elems);
    memset(dv, 0, sizeof(double) * n_sel * tile_elems);
    for (int32_t s = 0; s < n_sel; ++s) {
        const int32_t j = sel_tile[s];
        int32_t nq = 0;  /* query tiles whose list holds j at least once */
        for (int32_t i = 0; i < g.n_tiles; ++i)
            for (int32_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e)
                if (list[e] == j) {
                    q_list[nq++] = i;
                    break;
                }
        const double* qb = q + sel_bh[s] * slice;
        const double* kb = k + sel_bh[s] * slice;
        const double* vb = v + sel_bh[s] * slice;
        const double* dob = dout + sel_bh[s] * slice;
        double* dks = dk + s * tile_elems;
        double* dvs = dv + s * tile_elems;
#pragma omp parallel
        {
            int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * nk_max);
            double* P = (double*)malloc(sizeof(double) * nk_max);
            double* dP = (double*)malloc(sizeof(double) * nk_max);
            double* dk_local = (double*)calloc(tile_elems, sizeof(double));
            double* dv_local = (double*)calloc(tile_elems, sizeof(double));
            int ok = keys && P && dP && dk_local && dv_local;
            if (!ok) {
#pragma omp atomic write
                status = 2;
            }
#pragma omp for schedule(dynamic)
            for (int64_t job = 0; job < (int64_t)nq * g.tile_tokens; ++job) {
                if (!ok) continue;
                int32_t i = q_list[job / g.tile_tokens], r = (int32_t)(job % g.tile_tokens);
                int64_t nk = list_key_set(p, &g, row_ptr, list, i, keys);
                int64_t n = tile_token(p, &g, i, r);
                softmax_row(p, qb + n * p->d, kb, keys, nk, P);
                double D = 0.0;
                for (int64_t m = 0; m < nk; ++m) {
                    dP[m] = dot(dob + n * p->d, vb + keys[m] * p->d, p->d);
                    D += P[m] * dP[m];
                }
                for (int32_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
                    if (list[e] != j) continue;
                    const int64_t pos = e - row_ptr[i];  /* j's tokens are entries pos * tile_tokens + rk */
                    for (int32_t rk = 0; rk < g.tile_tokens; ++rk) {
                        int64_t m = pos * g.tile_tokens + rk;
                        double dS = P[m] * (dP[m] - D);
                        for (int32_t c = 0; c < p->d; ++c) {
                            dk_local[(int64_t)rk * p->d + c] += p->scale * dS * qb[n * p->d + c];
                            dv_local[(int64_t)rk * p->d + c] += P[m] * dob[n * p->d + c];
                        }
                    }
                }
            }
            if (ok) {
#pragma omp critical
                for (int64_t e = 0; e < tile_elems; ++e) {
                    dks[e] += dk_local[e];
                    dvs[e] += dv_local[e];
                }
            }
            free(keys);
            free(P);
            free(dP);
            free(dk_local);
            free(dv_local);
        }
    }
    free(q_list);
    return status;
}

/* ---------------------------------------------------------------------------------- */
/* Block attention mass (the sparsity map of a key-tile-list attention): for query tile i
 * and key tile j, the mean over the query tokens n of tile i of the attention probability
 * that n puts on the tokens of tile j,
 *     map[i][j] = (1 / tile_tokens) * sum_{n in i} sum over the positions of j's tokens in
 *                 K(i) of exp(s_nm - lse_n),
 * with K(i), lse_n as in oracle_fwd_list (a tile listed twice counts twice; tiles not
 * listed get 0; an empty list gives a zero row).  The rows of a non-empty list sum to one.
 * Selected (bh, query tile) pairs; map: [n_sel][nTiles]. */
int oracle_block_map_list(const oracle_problem* p, const double* q, const double* k, const int32_t* row_ptr,
                          const int32_t* list, int32_t n_sel, const int32_t* sel_bh, const int32_t* sel_tile,
                          double* map) {
    geometry g;
    if (make_geometry(p, &g) || check_lists(&g, row_ptr, list)) return 1;
    const int64_t nk_max = longest_list(&g, row_ptr) * g.tile_tokens + 1;
    const int64_t slice = (int64_t)g.n_tokens * p->d;
    int status = 0;
    memset(map, 0, sizeof(double) * n_sel * g.n_tiles);
#pragma omp parallel
    {
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * nk_max);
        double* P = (double*)malloc(sizeof(double) * nk_max);
        double* row = (double*)malloc(sizeof(double) * g.n_tiles);
        if (!keys || !P || !row) {
#pragma omp atomic write
            status = 2;
        }
#pragma omp for schedule(dynamic)
        for (int32_t s = 0; s < n_sel; ++s) {
            if (!keys || !P || !row) continue;
            const int32_t i = sel_tile[s];
            const double* qb = q + sel_bh[s] * slice;
            const double* kb = k + sel_bh[s] * slice;
            int64_t nk = list_key_set(p, &g, row_ptr, list, i, keys);
            for (int32_t j = 0; j < g.n_tiles; ++j) row[j] = 0.0;
            for (int32_t r = 0; r < g.tile_tokens && nk > 0; ++r) {
                int64_t n = tile_token(p, &g, i, r);
                softmax_row(p, qb + n * p->d, kb, keys, nk, P);
                for (int64_t m = 0; m < nk; ++m) row[list[row_ptr[i] + m / g.tile_tokens]] += P[m];
            }
            for (int32_t j = 0; j < g.n_tiles; ++j) map[(int64_t)s * g.n_tiles + j] = row[j] / g.tile_tokens;
        }
        free(keys);
        free(P);
        free(row);
    }
    return status;
}

/* ---------------------------------------------------------------------------------- */

/* Text prefix, video queries (the MOD-DiT page, "Token-Type-Aware Masking": text tokens
 * take part in full attention, only video-video attention is sparse).  Video query token
 * n of tile i attends to K(i) (its window, as oracle_fwd) and to every one of the L_text
 * text tokens, one softmax over the union:
 *     s_nm = scale <q_n, k_m> (m in K(i)),  s_nj = scale <q_n, k_text_j>,
 *     lse_n = ln (sum_m exp s_nm + sum_j exp s_nj),
 *     o_n = sum_m exp(s_nm - lse_n) v_m + sum_j exp(s_nj - lse_n) v_text_j.
 * k_text, v_text: [B*heads][L_text][d].  Selection and outputs as oracle_fwd. */
int oracle_fwd_prefix(const oracle_problem* p, const double* q, const double* k, const double* v,
                      const int32_t* offsets, int32_t L_text, const double* k_text, const double* v_text,
                      int32_t n_sel, const int32_t* sel_bh, const int32_t* sel_tile, double* out, double* lse) {
    geometry g;
    if (make_geometry(p, &g) || L_text < 0) return 1;
    const int64_t nw = (int64_t)g.n_window_tiles * g.tile_tokens;
    const int64_t slice = (int64_t)g.n_tokens * p->d, tslice = (int64_t)L_text * p->d;
    int status = 0;
#pragma omp parallel
    {
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * nw);
        double* P = (double*)malloc(sizeof(double) * (nw + L_text));
        if (!keys || !P) {
#pragma omp atomic write
            status = 2;
        }
#pragma omp for schedule(dynamic)
        for (int64_t job = 0; job < (int64_t)n_sel * g.tile_tokens; ++job) {
            if (!keys || !P) continue;
            int32_t s = (int32_t)(job / g.tile_tokens), r = (int32_t)(job % g.tile_tokens);
            const double* qb = q + sel_bh[s] * slice;
            const double* kb = k + sel_bh[s] * slice;
            const double* vb = v + sel_bh[s] * slice;
            const double* ktb = k_text + sel_bh[s] * tslice;
            const double* vtb = v_text + sel_bh[s] * tslice;
            key_set(p, &g, offsets, sel_tile[s], keys);
            const double* qn = qb + tile_token(p, &g, sel_tile[s], r) * p->d;
            /* scores over the union: window keys first, then the text keys */
            double mx = -INFINITY;
            for (int64_t m = 0; m < nw + L_text; ++m) {
                const double* km = m < nw ? kb + keys[m] * p->d : ktb + (m - nw) * p->d;
                P[m] = p->scale * dot(qn, km, p->d);
                if (P[m] > mx) mx = P[m];
            }
            double sum = 0.0;
            for (int64_t m = 0; m < nw + L_text; ++m) sum += exp(P[m] - mx);
            const double l = mx + log(sum);
            double* o = out + ((int64_t)s * g.tile_tokens + r) * p->d;
            for (int32_t c = 0; c < p->d; ++c) o[c] = 0.0;
            for (int64_t m = 0; m < nw + L_text; ++m) {
                const double w = exp(P[m] - l);
                const double* vm = m < nw ? vb + keys[m] * p->d : vtb + (m - nw) * p->d;
                for (int32_t c = 0; c < p->d; ++c) o[c] += w * vm[c];
            }
            lse[(int64_t)s * g.tile_tokens + r] = l;
        }
        free(keys);
        free(P);
    }
    return status;
}
