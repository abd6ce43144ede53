/*
 * Spatial Sparse Attention (SSA) -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, __graft_entry__.smoke() and the
 * benchmark's CPU-baseline leg may load this library. It shares no code, header,
 * table or helper with the CUDA library; the product path never calls it.
 *
 * What it computes (per sequence; sequences are independent):
 *   Direct3D-S2 model page (pixal-3d.com), "What is Direct3D-S2?": SSA partitions
 *   sparse tokens by their 3D coordinates and combines compressed global context,
 *   blockwise selection and local windows.
 *   Direct3D-S2 summary (nav.superapi.store), "Technical principles", SSA item:
 *   block-level tokens from a compression of each block; important blocks chosen
 *   from the compression module's attention scores; local window attention; the
 *   three outputs aggregated with predicted gating scores.
 * The concrete formulation (the pages leave it open) is:
 *   1. partition: block key (floor(x/8), floor(y/8), floor(z/8)); occupied blocks
 *      in lexicographic key order; tokens of a block in ascending index;
 *   2. compression: Kc_b = mean_{j in b}(K_j) . Wc, Vc_b likewise (row vector times
 *      the D x D matrix Wc, shared by K, V and all heads);
 *   3. compressed attention over all blocks of the sequence, softmax scale 1/sqrt(D);
 *   4. selection: own block plus the top (k-1) other blocks ranked by compressed
 *      logit (descending; equal logits -> lower block index); all blocks if Mb <= k;
 *   5. one softmax over all tokens of the selected blocks;
 *   6. window: one softmax over tokens j with max_axis |c_j - c_i| <= r (self
 *      included, blocks ignored);
 *   7. out = g0 * o_cmp + g1 * o_sel + g2 * o_win (gates given, not normalised).
 * Everything is accumulated in double. Inputs are decoded exactly from their
 * storage type (f32, bf16, f16). When `round_compressed` is set, Kc and Vc are
 * rounded (nearest-even) to the input type before use, modelling compressed
 * tokens stored in the input type so that block ranking is decided on the same
 * values on both sides.
 *
 * All functions are re-entrant; OpenMP parallelises over (row, head) pairs.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_F16 2
#define ORACLE_F64 3 /* test-only input type: lets finite differences run in full double */

/* ------------------------------------------------------------------------------------------ */
/* exact decoding of the storage types                                                         */
/* ------------------------------------------------------------------------------------------ */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_decode_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24); /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_decode_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void* base, int dtype, int64_t idx) {
    if (dtype == ORACLE_F64) return ((const double*)base)[idx];
    if (dtype == ORACLE_F32) return (double)((const float*)base)[idx];
    uint16_t h = ((const uint16_t*)base)[idx];
    return dtype == ORACLE_BF16 ? oracle_decode_bf16(h) : oracle_decode_f16(h);
}

/* Round x to the nearest value with `p` significant bits, minimum normal exponent `emin`
 * and largest finite value `maxv` (ties to even; overflow to infinity). */
static double round_to_format(double x, int p, int emin, double maxv) {
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    int e;
    frexp(x, &e);          /* |x| = m * 2^e, m in [0.5, 1): leading bit has exponent e-1 */
    int lead = e - 1;
    if (lead < emin) lead = emin; /* subnormal range: fixed spacing */
    double ulp = ldexp(1.0, lead - (p - 1));
    double q = nearbyint(x / ulp) * ulp; /* default rounding mode: nearest-even */
    if (fabs(q) > maxv) return x > 0 ? INFINITY : -INFINITY;
    return q;
}

double oracle_round_to(double x, int dtype) {
    switch (dtype) {
    case ORACLE_F64: return x;
    case ORACLE_F16: return round_to_format(x, 11, -14, 65504.0);
    case ORACLE_BF16: return round_to_format(x, 8, -126, ldexp(255.0, 120)); /* (2-2^-7)*2^127 */
    default: return round_to_format(x, 24, -126, ldexp(16777215.0, 104));  /* (2-2^-23)*2^127 */
    }
}

/* ------------------------------------------------------------------------------------------ */
/* 1. coordinate-block partition                                                               */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    int32_t bx, by, bz, idx;
} tok_key_t;

static int cmp_tok_key(const void* a, const void* b) {
    const tok_key_t* x = (const tok_key_t*)a;
    const tok_key_t* y = (const tok_key_t*)b;
    if (x->bx != y->bx) return x->bx < y->bx ? -1 : 1;
    if (x->by != y->by) return x->by < y->by ? -1 : 1;
    if (x->bz != y->bz) return x->bz < y->bz ? -1 : 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int32_t floor_div(int32_t a, int32_t b) {
    int32_t q = a / b;
    if ((a % b != 0) && ((a < 0) != (b < 0))) q -= 1;
    return q;
}

/* Groups the n tokens of one sequence into aligned block^3 blocks.
 * Outputs: perm[n] (tokens in block order, ascending index inside a block),
 * tok_blk[n] (block index of each token), blk_off[Mb+1], blk_coord[Mb*3].
 * Returns Mb (number of occupied blocks) or -1 on bad arguments. */
int64_t oracle_partition(int64_t n, const int32_t* coords, int32_t block, int32_t* perm,
                         int32_t* tok_blk, int32_t* blk_off, int32_t* blk_coord) {
    if (n < 0 || block <= 0) return -1;
    tok_key_t* keys = (tok_key_t*)malloc(sizeof(tok_key_t) * (size_t)(n > 0 ? n : 1));
    if (!keys) return -1;
    for (int64_t i = 0; i < n; ++i) {
        keys[i].bx = floor_div(coords[3 * i + 0], block);
        keys[i].by = floor_div(coords[3 * i + 1], block);
        keys[i].bz = floor_div(coords[3 * i + 2], block);
        keys[i].idx = (int32_t)i;
    }
    qsort(keys, (size_t)n, sizeof(tok_key_t), cmp_tok_key);
    int64_t mb = 0;
    for (int64_t p = 0; p < n; ++p) {
        int new_block = (p == 0) || keys[p].bx != keys[p - 1].bx || keys[p].by != keys[p - 1].by ||
                        keys[p].bz != keys[p - 1].bz;
        if (new_block) {
            blk_off[mb] = (int32_t)p;
            blk_coord[3 * mb + 0] = keys[p].bx;
            blk_coord[3 * mb + 1] = keys[p].by;
            blk_coord[3 * mb + 2] = keys[p].bz;
            mb += 1;
        }
        perm[p] = keys[p].idx;
        tok_blk[keys[p].idx] = (int32_t)(mb - 1);
    }
    blk_off[mb] = (int32_t)n;
    free(keys);
    return mb;
}

/* ------------------------------------------------------------------------------------------ */
/* 6a. window neighbour lists                                                                  */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    int32_t x, y, z, idx;
} cell_t;

static int cmp_cell(const void* a, const void* b) {
    const cell_t* p = (const cell_t*)a;
    const cell_t* q = (const cell_t*)b;
    if (p->x != q->x) return p->x < q->x ? -1 : 1;
    if (p->y != q->y) return p->y < q->y ? -1 : 1;
    if (p->z != q->z) return p->z < q->z ? -1 : 1;
    return (p->idx > q->idx) - (p->idx < q->idx);
}

static int cmp_i32(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

static int64_t find_cell(const cell_t* cells, int64_t n, int32_t x, int32_t y, int32_t z) {
    int64_t lo = 0, hi = n;
    while (lo < hi) {
        int64_t mid = lo + (hi - lo) / 2;
        const cell_t* c = &cells[mid];
        int less = c->x < x || (c->x == x && (c->y < y || (c->y == y && c->z < z)));
        if (less) lo = mid + 1; else hi = mid;
    }
    if (lo < n && cells[lo].x == x && cells[lo].y == y && cells[lo].z == z) return lo;
    return -1;
}

/* Window W(i) = { j : max(|x_j-x_i|, |y_j-y_i|, |z_j-z_i|) <= r }, self included, found by
 * looking up every cell of the (2r+1)^3 cube around c_i. Coordinates must be unique.
 * If nbr_idx is NULL only counts are produced: nbr_off[0..n] gets the CSR offsets and the
 * return value is nnz. Otherwise nbr_idx is filled, each row in ascending index order.
 * Returns -2 if two tokens share a coordinate. */
int64_t oracle_window(int64_t n, const int32_t* coords, int32_t r, int64_t* nbr_off,
                      int32_t* nbr_idx) {
    cell_t* cells = (cell_t*)malloc(sizeof(cell_t) * (size_t)(n > 0 ? n : 1));
    if (!cells) return -1;
    for (int64_t i = 0; i < n; ++i) {
        cells[i].x = coords[3 * i];
        cells[i].y = coords[3 * i + 1];
        cells[i].z = coords[3 * i + 2];
        cells[i].idx = (int32_t)i;
    }
    qsort(cells, (size_t)n, sizeof(cell_t), cmp_cell);
    for (int64_t p = 1; p < n; ++p) {
        if (cells[p].x == cells[p - 1].x && cells[p].y == cells[p - 1].y &&
            cells[p].z == cells[p - 1].z) {
            free(cells);
            return -2;
        }
    }
    int64_t total = 0;
    if (!nbr_idx) nbr_off[0] = 0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t cnt = 0;
        int32_t* row = nbr_idx ? nbr_idx + nbr_off[i] : NULL;
        for (int32_t dx = -r; dx <= r; ++dx)
            for (int32_t dy = -r; dy <= r; ++dy)
                for (int32_t dz = -r; dz <= r; ++dz) {
                    int64_t at = find_cell(cells, n, coords[3 * i] + dx, coords[3 * i + 1] + dy,
                                           coords[3 * i + 2] + dz);
                    if (at >= 0) {
                        if (row) row[cnt] = cells[at].idx;
                        cnt += 1;
                    }
                }
        if (row) qsort(row, (size_t)cnt, sizeof(int32_t), cmp_i32);
        total += cnt;
        if (!nbr_idx) nbr_off[i + 1] = total;
    }
    free(cells);
    return total;
}

/* Brute force over all pairs, for tiny inputs: same contract as oracle_window. */
int64_t oracle_window_brute(int64_t n, const int32_t* coords, int32_t r, int64_t* nbr_off,
                            int32_t* nbr_idx) {
    int64_t total = 0;
    if (!nbr_idx) nbr_off[0] = 0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t cnt = 0;
        for (int64_t j = 0; j < n; ++j) {
            int32_t d = abs(coords[3 * j] - coords[3 * i]);
            int32_t dy = abs(coords[3 * j + 1] - coords[3 * i + 1]);
            int32_t dz = abs(coords[3 * j + 2] - coords[3 * i + 2]);
            if (dy > d) d = dy;
            if (dz > d) d = dz;
            if (d <= r) {
                if (nbr_idx) nbr_idx[nbr_off[i] + cnt] = (int32_t)j;
                cnt += 1;
            }
        }
        total += cnt;
        if (!nbr_idx) nbr_off[i + 1] = total;
    }
    return total;
}

/* ------------------------------------------------------------------------------------------ */
/* 2. compression                                                                              */
/* ------------------------------------------------------------------------------------------ */

/* Kc[b][h][e] = sum_d mean_{j in b}(K[j][h][d]) * Wc[d][e]; same for V. Layout [Mb, H, D]. */
static void compress(int64_t mb, int32_t H, int32_t D, int dtype, const void* K, const void* V,
                     const float* Wc, const int32_t* perm, const int32_t* blk_off,
                     int round_compressed, double* Kc, double* Vc) {
#pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < mb * H; ++bh) {
        int64_t b = bh / H;
        int32_t h = (int32_t)(bh % H);
        int64_t nb = blk_off[b + 1] - blk_off[b];
        double* kmean = (double*)calloc((size_t)D, sizeof(double));
        double* vmean = (double*)calloc((size_t)D, sizeof(double));
        for (int64_t p = blk_off[b]; p < blk_off[b + 1]; ++p) {
            int64_t j = perm[p];
            for (int32_t d = 0; d < D; ++d) {
                kmean[d] += load_elem(K, dtype, (j * H + h) * D + d);
                vmean[d] += load_elem(V, dtype, (j * H + h) * D + d);
            }
        }
        for (int32_t d = 0; d < D; ++d) {
            kmean[d] /= (double)nb;
            vmean[d] /= (double)nb;
        }
        for (int32_t e = 0; e < D; ++e) {
            double sk = 0.0, sv = 0.0;
            for (int32_t d = 0; d < D; ++d) {
                sk += kmean[d] * (double)Wc[d * D + e];
                sv += vmean[d] * (double)Wc[d * D + e];
            }
            if (round_compressed) {
                sk = oracle_round_to(sk, dtype);
                sv = oracle_round_to(sv, dtype);
            }
            Kc[(b * H + h) * D + e] = sk;
            Vc[(b * H + h) * D + e] = sv;
        }
        free(kmean);
        free(vmean);
    }
}

/* Exported for tests: the compressed tokens of one sequence, [Mb, H, D] each. */
int oracle_compress(int64_t mb, int32_t H, int32_t D, int32_t dtype, const void* K, const void* V,
                    const float* Wc, const int32_t* perm, const int32_t* blk_off,
                    int32_t round_compressed, double* Kc, double* Vc) {
    compress(mb, H, D, dtype, K, V, Wc, perm, blk_off, round_compressed, Kc, Vc);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* 2b. compression by a sparse 3D convolution over the block grid                              */
/* ------------------------------------------------------------------------------------------ */

/*
 * Direct3D-S2 summary page, "Technical principles of Direct3D-S2", SSA item: the compression
 * module turns each block into a block-level token by sparse 3D convolution and pooling. The
 * page gives no shapes; the plain reading taken here: pool first (the mean over the tokens
 * present in the block, as in step 2), then one sparse 3D convolution over the grid of occupied
 * blocks with a 3x3x3 kernel, stride 1, outputs at the occupied blocks only, an absent
 * neighbour contributing nothing:
 *   Kc_b = sum over offsets o in {-1,0,1}^3 with block b+o occupied of mean(K_{b+o}) . W_o
 * W_o (D x D, row vector times W_o) is shared by K, V and all heads; offset (dx, dy, dz) is
 * W[9*(dx+1) + 3*(dy+1) + (dz+1)]. With W_o = 0 except W_0 = Wc this is step 2.
 */

/* Index of the block of one sequence with block coordinates (x, y, z), or -1 (blk_coord holds
 * the occupied blocks in lexicographic order). */
static int64_t find_block(const int32_t* blk_coord, int64_t mb, int32_t x, int32_t y, int32_t z) {
    int64_t lo = 0, hi = mb;
    while (lo < hi) {
        int64_t mid = lo + (hi - lo) / 2;
        const int32_t* c = &blk_coord[3 * mid];
        int less = c[0] < x || (c[0] == x && (c[1] < y || (c[1] == y && c[2] < z)));
        if (less) lo = mid + 1; else hi = mid;
    }
    if (lo < mb && blk_coord[3 * lo] == x && blk_coord[3 * lo + 1] == y && blk_coord[3 * lo + 2] == z)
        return lo;
    return -1;
}

static void compress_conv(int64_t mb, int32_t H, int32_t D, int dtype, const void* K, const void* V,
                          const float* W, const int32_t* perm, const int32_t* blk_off,
                          const int32_t* blk_coord, double* Kc, double* Vc) {
    double* km = (double*)calloc((size_t)(mb * H * D + 1), sizeof(double));
    double* vm = (double*)calloc((size_t)(mb * H * D + 1), sizeof(double));
#pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < mb * H; ++bh) {
        int64_t b = bh / H;
        int32_t h = (int32_t)(bh % H);
        int64_t nb = blk_off[b + 1] - blk_off[b];
        for (int64_t p = blk_off[b]; p < blk_off[b + 1]; ++p) {
            int64_t j = perm[p];
            for (int32_t d = 0; d < D; ++d) {
                km[bh * D + d] += load_elem(K, dtype, (j * H + h) * D + d);
                vm[bh * D + d] += load_elem(V, dtype, (j * H + h) * D + d);
            }
        }
        for (int32_t d = 0; d < D; ++d) {
            km[bh * D + d] /= (double)nb;
            vm[bh * D + d] /= (double)nb;
        }
    }
#pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < mb * H; ++bh) {
        int64_t b = bh / H;
        int32_t h = (int32_t)(bh % H);
        for (int32_t e = 0; e < D; ++e) {
            Kc[bh * D + e] = 0.0;
            Vc[bh * D + e] = 0.0;
        }
        for (int32_t o = 0; o < 27; ++o) {
            int64_t nb = find_block(blk_coord, mb, blk_coord[3 * b] + o / 9 - 1,
                                    blk_coord[3 * b + 1] + (o / 3) % 3 - 1, blk_coord[3 * b + 2] + o % 3 - 1);
            if (nb < 0) continue;
            const double* mk = &km[(nb * H + h) * D];
            const double* mv = &vm[(nb * H + h) * D];
            const float* Wo = &W[(int64_t)o * D * D];
            for (int32_t e = 0; e < D; ++e) {
                double sk = 0.0, sv = 0.0;
                for (int32_t d = 0; d < D; ++d) {
                    sk += mk[d] * (double)Wo[d * D + e];
                    sv += mv[d] * (double)Wo[d * D + e];
                }
                Kc[bh * D + e] += sk;
                Vc[bh * D + e] += sv;
            }
        }
    }
    free(km);
    free(vm);
}

/* Exported for tests: the convolution-compressed tokens of one sequence, [Mb, H, D] each. */
int oracle_compress_conv(int64_t mb, int32_t H, int32_t D, int32_t dtype, const void* K, const void* V,
                         const float* W, const int32_t* perm, const int32_t* blk_off,
                         const int32_t* blk_coord, double* Kc, double* Vc) {
    compress_conv(mb, H, D, dtype, K, V, W, perm, blk_off, blk_coord, Kc, Vc);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* 3-7. forward for a set of query rows                                                        */
/* ------------------------------------------------------------------------------------------ */

/* softmax attention of query q (length D) over `nk` keys given as row pointers.
 * Writes o[D] = sum_j softmax(scale * q.k_j)_j * v_j. */
static void attend(int32_t D, const double* q, int64_t nk, const double* const* krow,
                   const double* const* vrow, double scale, double* logits, double* o) {
    double m = -INFINITY;
    for (int64_t j = 0; j < nk; ++j) {
        double z = 0.0;
        for (int32_t d = 0; d < D; ++d) z += q[d] * krow[j][d];
        logits[j] = scale * z;
        if (logits[j] > m) m = logits[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < nk; ++j) {
        logits[j] = exp(logits[j] - m);
        l += logits[j];
    }
    for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < nk; ++j) {
        double p = logits[j] / l;
        for (int32_t d = 0; d < D; ++d) o[d] += p * vrow[j][d];
    }
}

/* Rank the blocks other than `own` by compressed logit z (descending, equal -> lower index)
 * and fill sel[0..k-1]: sel[0] = own, then the best k-1 others; -1 where fewer exist. */
static void select_blocks(int64_t mb, const double* z, int32_t own, int32_t k, int32_t* sel) {
    for (int32_t s = 0; s < k; ++s) sel[s] = -1;
    sel[0] = own;
    for (int32_t s = 1; s < k; ++s) {
        int32_t best = -1;
        for (int64_t b = 0; b < mb; ++b) {
            if (b == own) continue;
            int taken = 0;
            for (int32_t t = 1; t < s; ++t) taken |= (sel[t] == b);
            if (taken) continue;
            if (best < 0 || z[b] > z[best]) best = (int32_t)b; /* strict: lower index wins ties */
        }
        sel[s] = best;
        if (best < 0) break;
    }
}

/*
 * 4b. Selection shared by the queries of one 4x4x4 sub-block of cells.
 * The pages choose the important blocks from the compression module's attention scores and
 * leave open whose scores (Direct3D-S2 summary page, "Technical principles", SSA item). This
 * variant pools them over a sub-block G = the tokens of the sequence with the same
 * (floor(x/4), floor(y/4), floor(z/4)); as 4 divides 8, G lies in one block, its members' own
 * block. Per head:
 *   score_G(b) = sum_{i in G} p_i(b),  p_i = softmax_b(scale * q_i . Kc_b)  (step 3's weights);
 *   every member of G takes S_G = {own} + the top (k-1) other blocks by score_G (descending,
 *   equal scores -> lower block index), ranked by select_blocks.
 * coords: [n, 3] of the sequence (non-negative). Compression as the forward: Kc from Wconv
 * (section 2b) when non-NULL, else mean . Wc, unrounded. Outputs for the `n_rows` rows (local
 * indices in `rows`; NULL = all n): sel [n_rows, H, k] local block indices (-1 = empty slot),
 * and score (may be NULL) [n_rows, H, mb] = score_G of the row's sub-block.
 */
static int32_t subblock_of(const int32_t* c) {
    return (((c[0] >> 2) & 1) << 2) | (((c[1] >> 2) & 1) << 1) | ((c[2] >> 2) & 1);
}

int oracle_select_subblock(int64_t n, int32_t H, int32_t D, int32_t dtype, const void* Q,
                           const void* K, const void* V, const float* Wc, const float* Wconv,
                           const int32_t* blk_coord, int32_t topk, const int32_t* coords,
                           const int32_t* perm, const int32_t* tok_blk, const int32_t* blk_off,
                           int64_t mb, int64_t n_rows, const int64_t* rows, int32_t* sel,
                           double* score) {
    if (topk < 1 || D < 1 || H < 1 || mb < 1) return -1;
    if (!rows) n_rows = n;
    const int64_t ng = mb * 8; /* group id = 8 * block + sub-block of the block */
    int64_t* g_off = (int64_t*)calloc((size_t)(ng + 1), sizeof(int64_t));
    int64_t* g_mem = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n + 1));
    int64_t* g_slot = (int64_t*)malloc(sizeof(int64_t) * (size_t)(ng + 1)); /* needed group -> slot */
    double* Kc = (double*)malloc(sizeof(double) * (size_t)(mb * H * D + 1));
    double* Vc = (double*)malloc(sizeof(double) * (size_t)(mb * H * D + 1));
    if (!g_off || !g_mem || !g_slot || !Kc || !Vc) return -1;
    if (Wconv)
        compress_conv(mb, H, D, dtype, K, V, Wconv, perm, blk_off, blk_coord, Kc, Vc);
    else
        compress(mb, H, D, dtype, K, V, Wc, perm, blk_off, 0, Kc, Vc);
    /* members of every group, in ascending token index */
    for (int64_t i = 0; i < n; ++i) g_off[8 * (int64_t)tok_blk[i] + subblock_of(&coords[3 * i]) + 1] += 1;
    for (int64_t g = 0; g < ng; ++g) g_off[g + 1] += g_off[g];
    {
        int64_t* fill = (int64_t*)malloc(sizeof(int64_t) * (size_t)(ng + 1));
        if (!fill) return -1;
        memcpy(fill, g_off, sizeof(int64_t) * (size_t)ng);
        for (int64_t i = 0; i < n; ++i) g_mem[fill[8 * (int64_t)tok_blk[i] + subblock_of(&coords[3 * i])]++] = i;
        free(fill);
    }
    /* the groups the requested rows belong to */
    for (int64_t g = 0; g < ng; ++g) g_slot[g] = -1;
    int64_t n_need = 0;
    for (int64_t ri = 0; ri < n_rows; ++ri) {
        int64_t i = rows ? rows[ri] : ri;
        int64_t g = 8 * (int64_t)tok_blk[i] + subblock_of(&coords[3 * i]);
        if (g_slot[g] < 0) g_slot[g] = n_need++;
    }
    int64_t* need = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_need + 1));
    int32_t* gsel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_need * H * topk + 1));
    double* gscore = score ? (double*)malloc(sizeof(double) * (size_t)(n_need * H * mb + 1)) : NULL;
    if (!need || !gsel || (score && !gscore)) return -1;
    for (int64_t g = 0; g < ng; ++g)
        if (g_slot[g] >= 0) need[g_slot[g]] = g;
    const double scale = 1.0 / sqrt((double)D);

#pragma omp parallel
    {
        double* q = (double*)malloc(sizeof(double) * (size_t)D);
        double* z = (double*)malloc(sizeof(double) * (size_t)mb);
        double* acc = (double*)malloc(sizeof(double) * (size_t)mb);
#pragma omp for schedule(dynamic, 4)
        for (int64_t gh = 0; gh < n_need * H; ++gh) {
            const int64_t slot = gh / H, g = need[slot];
            const int32_t h = (int32_t)(gh % H);
            for (int64_t b = 0; b < mb; ++b) acc[b] = 0.0;
            for (int64_t t = g_off[g]; t < g_off[g + 1]; ++t) {
                const int64_t i = g_mem[t];
                for (int32_t d = 0; d < D; ++d) q[d] = load_elem(Q, dtype, (i * H + h) * D + d);
                /* this member's compressed-attention weights, as in step 3 */
                double m = -INFINITY;
                for (int64_t b = 0; b < mb; ++b) {
                    double t2 = 0.0;
                    for (int32_t d = 0; d < D; ++d) t2 += q[d] * Kc[(b * H + h) * D + d];
                    z[b] = scale * t2;
                    if (z[b] > m) m = z[b];
                }
                double l = 0.0;
                for (int64_t b = 0; b < mb; ++b) {
                    z[b] = exp(z[b] - m);
                    l += z[b];
                }
                for (int64_t b = 0; b < mb; ++b) acc[b] += z[b] / l;
            }
            select_blocks(mb, acc, (int32_t)(g / 8), topk, &gsel[gh * topk]);
            if (gscore)
                for (int64_t b = 0; b < mb; ++b) gscore[gh * mb + b] = acc[b];
        }
        free(q); free(z); free(acc);
    }
    for (int64_t ri = 0; ri < n_rows; ++ri) {
        int64_t i = rows ? rows[ri] : ri;
        int64_t slot = g_slot[8 * (int64_t)tok_blk[i] + subblock_of(&coords[3 * i])];
        for (int32_t h = 0; h < H; ++h) {
            for (int32_t s2 = 0; s2 < topk; ++s2)
                sel[(ri * H + h) * topk + s2] = gsel[(slot * H + h) * topk + s2];
            if (score)
                for (int64_t b = 0; b < mb; ++b) score[(ri * H + h) * mb + b] = gscore[(slot * H + h) * mb + b];
        }
    }
    free(g_off); free(g_mem); free(g_slot); free(need); free(gsel); free(gscore); free(Kc); free(Vc);
    return 0;
}

/*
 * Forward pass of one sequence for `n_rows` query rows (local indices in `rows`; NULL = all n).
 * Q, K, V: [n, H, D] of `dtype`; gates: [n, H, 3] (cmp, sel, win); Wc: [D, D].
 * Plan arrays come from oracle_partition / oracle_window of the same sequence.
 * Outputs (each may be NULL), per evaluated row:
 *   out, o_cmp, o_sel, o_win: [n_rows, H, D];  sel: [n_rows, H, k] (local block indices);
 *   zc: [n_rows, H, Mb] scaled compressed logits.
 * If sel_in is non-NULL ([n_rows, H, k], -1 = empty slot) it replaces the computed selection
 * (used by tests to pin the selection branch with planted block sets, and to evaluate the
 * branches with another implementation's validated choice among near-tied blocks).
 * When out, o_sel and o_win are all NULL only steps 3-4 run (compressed attention and the
 * selection), so the selection of many rows can be had at the cost of the compressed branch.
 */
static int forward_impl(int64_t n, int32_t H, int32_t D, int32_t dtype, const void* Q, const void* K,
                        const void* V, const float* gates, const float* Wc, int32_t topk,
                        int32_t round_compressed, const int32_t* perm, const int32_t* tok_blk,
                        const int32_t* blk_off, int64_t mb, const int64_t* nbr_off,
                        const int32_t* nbr_idx, int64_t n_rows, const int64_t* rows,
                        const int32_t* sel_in, double* out, double* o_cmp, double* o_sel,
                        double* o_win, int32_t* sel, double* zc, const float* Wconv,
                        const int32_t* blk_coord, const float* Wg, const float* bg) {
    if (topk < 1 || D < 1 || H < 1) return -1;
    if (!rows) n_rows = n;
    double* Kc = (double*)malloc(sizeof(double) * (size_t)(mb * H * D + 1));
    double* Vc = (double*)malloc(sizeof(double) * (size_t)(mb * H * D + 1));
    if (!Kc || !Vc) return -1;
    if (Wconv)
        compress_conv(mb, H, D, dtype, K, V, Wconv, perm, blk_off, blk_coord, Kc, Vc);
    else
        compress(mb, H, D, dtype, K, V, Wc, perm, blk_off, round_compressed, Kc, Vc);
    const double scale = 1.0 / sqrt((double)D);
    int64_t max_nb = 0;
    for (int64_t b = 0; b < mb; ++b)
        if (blk_off[b + 1] - blk_off[b] > max_nb) max_nb = blk_off[b + 1] - blk_off[b];
    int64_t max_win = 0;
    for (int64_t i = 0; i < n; ++i)
        if (nbr_off[i + 1] - nbr_off[i] > max_win) max_win = nbr_off[i + 1] - nbr_off[i];
    int64_t max_keys = max_nb * topk;
    if (max_win > max_keys) max_keys = max_win;
    if (mb > max_keys) max_keys = mb;

#pragma omp parallel
    {
        double* q = (double*)malloc(sizeof(double) * (size_t)D);
        double* oc = (double*)malloc(sizeof(double) * (size_t)D);
        double* os = (double*)malloc(sizeof(double) * (size_t)D);
        double* ow = (double*)malloc(sizeof(double) * (size_t)D);
        double* logits = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1));
        double* z = (double*)malloc(sizeof(double) * (size_t)(mb + 1));
        int32_t* s_loc = (int32_t*)malloc(sizeof(int32_t) * (size_t)topk);
        double* kbuf = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1) * (size_t)D);
        double* vbuf = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1) * (size_t)D);
        const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(max_keys + 1));
        const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(max_keys + 1));

#pragma omp for schedule(dynamic, 4)
        for (int64_t rh = 0; rh < n_rows * H; ++rh) {
            int64_t ri = rh / H;
            int32_t h = (int32_t)(rh % H);
            int64_t i = rows ? rows[ri] : ri;
            for (int32_t d = 0; d < D; ++d) q[d] = load_elem(Q, dtype, (i * H + h) * D + d);

            /* 3. compressed attention over every block of the sequence */
            for (int64_t b = 0; b < mb; ++b) {
                kr[b] = &Kc[(b * H + h) * D];
                vr[b] = &Vc[(b * H + h) * D];
            }
            attend(D, q, mb, kr, vr, scale, logits, oc);
            for (int64_t b = 0; b < mb; ++b) {
                double t = 0.0;
                for (int32_t d = 0; d < D; ++d) t += q[d] * Kc[(b * H + h) * D + d];
                z[b] = scale * t;
            }
            if (zc)
                for (int64_t b = 0; b < mb; ++b) zc[(ri * H + h) * mb + b] = z[b];

            /* 4. selection: own block + top (k-1) others by compressed logit */
            if (sel_in) {
                for (int32_t s = 0; s < topk; ++s) s_loc[s] = sel_in[(ri * H + h) * topk + s];
            } else {
                select_blocks(mb, z, tok_blk[i], topk, s_loc);
            }
            if (sel)
                for (int32_t s = 0; s < topk; ++s) sel[(ri * H + h) * topk + s] = s_loc[s];

            /* selection only (no branch output requested): steps 5-7 are not needed */
            if (!out && !o_sel && !o_win) {
                if (o_cmp)
                    for (int32_t d = 0; d < D; ++d) o_cmp[(ri * H + h) * D + d] = oc[d];
                continue;
            }

            /* 5. one softmax over the tokens of all selected blocks */
            int64_t nk = 0;
            for (int32_t s = 0; s < topk; ++s) {
                int32_t b = s_loc[s];
                if (b < 0) continue;
                for (int64_t p = blk_off[b]; p < blk_off[b + 1]; ++p) {
                    int64_t j = perm[p];
                    for (int32_t d = 0; d < D; ++d) {
                        kbuf[nk * D + d] = load_elem(K, dtype, (j * H + h) * D + d);
                        vbuf[nk * D + d] = load_elem(V, dtype, (j * H + h) * D + d);
                    }
                    kr[nk] = &kbuf[nk * D];
                    vr[nk] = &vbuf[nk * D];
                    nk += 1;
                }
            }
            attend(D, q, nk, kr, vr, scale, logits, os);

            /* 6. window: tokens within Chebyshev radius r */
            nk = 0;
            for (int64_t t = nbr_off[i]; t < nbr_off[i + 1]; ++t) {
                int64_t j = nbr_idx[t];
                for (int32_t d = 0; d < D; ++d) {
                    kbuf[nk * D + d] = load_elem(K, dtype, (j * H + h) * D + d);
                    vbuf[nk * D + d] = load_elem(V, dtype, (j * H + h) * D + d);
                }
                kr[nk] = &kbuf[nk * D];
                vr[nk] = &vbuf[nk * D];
                nk += 1;
            }
            attend(D, q, nk, kr, vr, scale, logits, ow);

            /* 7. gated sum; with a gate predictor, g_c = sigmoid(bg_c + sum_d q_d Wg[d][c]) */
            double g[3];
            for (int32_t c = 0; c < 3; ++c) {
                if (Wg) {
                    double t = (double)bg[c];
                    for (int32_t d = 0; d < D; ++d) t += q[d] * (double)Wg[d * 3 + c];
                    g[c] = 1.0 / (1.0 + exp(-t));
                } else {
                    g[c] = (double)gates[(i * H + h) * 3 + c];
                }
            }
            for (int32_t d = 0; d < D; ++d) {
                int64_t o = (ri * H + h) * D + d;
                if (o_cmp) o_cmp[o] = oc[d];
                if (o_sel) o_sel[o] = os[d];
                if (o_win) o_win[o] = ow[d];
                if (out) out[o] = g[0] * oc[d] + g[1] * os[d] + g[2] * ow[d];
            }
        }
        free(q); free(oc); free(os); free(ow); free(logits); free(z); free(s_loc);
        free(kbuf); free(vbuf); free(kr); free(vr);
    }
    free(Kc);
    free(Vc);
    return 0;
}

int oracle_forward(int64_t n, int32_t H, int32_t D, int32_t dtype, const void* Q, const void* K,
                   const void* V, const float* gates, const float* Wc, int32_t topk,
                   int32_t round_compressed, const int32_t* perm, const int32_t* tok_blk,
                   const int32_t* blk_off, int64_t mb, const int64_t* nbr_off,
                   const int32_t* nbr_idx, int64_t n_rows, const int64_t* rows,
                   const int32_t* sel_in, double* out, double* o_cmp, double* o_sel,
                   double* o_win, int32_t* sel, double* zc) {
    return forward_impl(n, H, D, dtype, Q, K, V, gates, Wc, topk, round_compressed, perm, tok_blk,
                        blk_off, mb, nbr_off, nbr_idx, n_rows, rows, sel_in, out, o_cmp, o_sel,
                        o_win, sel, zc, NULL, NULL, NULL, NULL);
}

/*
 * The forward with the compression by sparse 3D convolution (section 2b; Wconv [27, D, D],
 * blk_coord [Mb, 3] of the sequence) and, when Wg is non-NULL, the gates predicted from each
 * head's query (Direct3D-S2 summary page, "Technical principles", SSA item: the branches are
 * aggregated with predicted gating scores): g = sigmoid(q . Wg + bg), Wg [D, 3], bg [3], shared
 * by all heads, in the order (cmp, sel, win); `gates` is then not read. Other arguments as
 * oracle_forward.
 */
int oracle_forward_variant(int64_t n, int32_t H, int32_t D, int32_t dtype, const void* Q,
                           const void* K, const void* V, const float* gates, const float* Wconv,
                           const int32_t* blk_coord, const float* Wg, const float* bg, int32_t topk,
                           const int32_t* perm, const int32_t* tok_blk, const int32_t* blk_off,
                           int64_t mb, const int64_t* nbr_off, const int32_t* nbr_idx,
                           int64_t n_rows, const int64_t* rows, const int32_t* sel_in, double* out,
                           double* o_cmp, double* o_sel, double* o_win, int32_t* sel, double* zc) {
    if (!Wconv || !blk_coord) return -1;
    return forward_impl(n, H, D, dtype, Q, K, V, gates, NULL, topk, 0, perm, tok_blk, blk_off, mb,
                        nbr_off, nbr_idx, n_rows, rows, sel_in, out, o_cmp, o_sel, o_win, sel, zc,
                        Wconv, blk_coord, Wg, bg);
}

/* ------------------------------------------------------------------------------------------ */
/* 8. backward                                                                                 */
/* ------------------------------------------------------------------------------------------ */

/*
 * Gradient of one attention branch for one (row, head), given its key/value rows.
 * With z_j = scale * q.k_j, P = softmax(z), o = sum_j P_j v_j and branch output weighted by g:
 *   dP_j = g * dO . v_j;  dz_j = P_j * (dP_j - sum_t P_t dP_t)
 *   dq  += scale * sum_j dz_j k_j;  dk_j += scale * dz_j q;  dv_j += g * P_j dO.
 * dk/dv are written to per-key scratch rows (dkr[j], dvr[j]) by accumulation.
 */
static void attend_backward(int32_t D, const double* q, const double* dO, double g, int64_t nk,
                            const double* const* krow, const double* const* vrow, double scale,
                            double* P, double* dP, double* dq, double* const* dkr,
                            double* const* dvr) {
    double m = -INFINITY;
    for (int64_t j = 0; j < nk; ++j) {
        double z = 0.0;
        for (int32_t d = 0; d < D; ++d) z += q[d] * krow[j][d];
        P[j] = scale * z;
        if (P[j] > m) m = P[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < nk; ++j) {
        P[j] = exp(P[j] - m);
        l += P[j];
    }
    double pdp = 0.0;
    for (int64_t j = 0; j < nk; ++j) {
        P[j] /= l;
        double t = 0.0;
        for (int32_t d = 0; d < D; ++d) t += dO[d] * vrow[j][d];
        dP[j] = g * t;
        pdp += P[j] * dP[j];
    }
    for (int64_t j = 0; j < nk; ++j) {
        double dz = P[j] * (dP[j] - pdp);
        for (int32_t d = 0; d < D; ++d) {
            dq[d] += scale * dz * krow[j][d];
            if (dkr) dkr[j][d] += scale * dz * q[d];
            if (dvr) dvr[j][d] += g * P[j] * dO[d];
        }
    }
}

/*
 * Full backward of one sequence: dQ, dK, dV [n, H, D] (double) of
 *   L = sum_{i,h,d} dO[i,h,d] * out[i,h,d]
 * with the selection held at `sel` ([n, H, k], local block indices, as produced by
 * oracle_forward for all rows) and the compressed tokens' rounding treated as identity.
 * Compression: dK_j += (1/n_b) * (dKc_b . Wc^T) for every token j of block b; same for V.
 * Heads are independent and are taken one after the other. Inside a head the query rows are
 * shared among the threads; each thread adds its rows' key and value gradients into its own
 * zeroed copy of dK, dV, dKc, dVc, and the copies are summed in thread order at the end.
 */
int oracle_backward(int64_t n, int32_t H, int32_t D, int32_t dtype, const void* Q, const void* K,
                    const void* V, const float* gates, const float* Wc, const void* dO,
                    int32_t topk, int32_t round_compressed, const int32_t* perm,
                    const int32_t* tok_blk, const int32_t* blk_off, int64_t mb,
                    const int64_t* nbr_off, const int32_t* nbr_idx, const int32_t* sel,
                    double* dQ, double* dK, double* dV) {
    (void)tok_blk;
    double* Kc = (double*)malloc(sizeof(double) * (size_t)(mb * H * D + 1));
    double* Vc = (double*)malloc(sizeof(double) * (size_t)(mb * H * D + 1));
    if (!Kc || !Vc) return -1;
    compress(mb, H, D, dtype, K, V, Wc, perm, blk_off, round_compressed, Kc, Vc);
    const double scale = 1.0 / sqrt((double)D);
    memset(dQ, 0, sizeof(double) * (size_t)(n * H * D));
    memset(dK, 0, sizeof(double) * (size_t)(n * H * D));
    memset(dV, 0, sizeof(double) * (size_t)(n * H * D));
    int64_t max_nb = 0;
    for (int64_t b = 0; b < mb; ++b)
        if (blk_off[b + 1] - blk_off[b] > max_nb) max_nb = blk_off[b + 1] - blk_off[b];
    int64_t max_keys = max_nb * topk;
    for (int64_t i = 0; i < n; ++i)
        if (nbr_off[i + 1] - nbr_off[i] > max_keys) max_keys = nbr_off[i + 1] - nbr_off[i];
    if (mb > max_keys) max_keys = mb;

    const int nt = omp_get_max_threads();
    const size_t tok_elems = (size_t)(n * D + 1), blk_elems = (size_t)(mb * D + 1);
    double* kall = (double*)malloc(sizeof(double) * tok_elems);
    double* vall = (double*)malloc(sizeof(double) * tok_elems);
    double* dkall = (double*)malloc(sizeof(double) * tok_elems * (size_t)nt);  /* one per thread */
    double* dvall = (double*)malloc(sizeof(double) * tok_elems * (size_t)nt);
    double* dKc = (double*)malloc(sizeof(double) * blk_elems * (size_t)nt);
    double* dVc = (double*)malloc(sizeof(double) * blk_elems * (size_t)nt);
    if (!kall || !vall || !dkall || !dvall || !dKc || !dVc) {
        free(Kc); free(Vc); free(kall); free(vall); free(dkall); free(dvall); free(dKc); free(dVc);
        return -1;
    }

    for (int32_t h = 0; h < H; ++h) {
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < n; ++j)
            for (int32_t d = 0; d < D; ++d) {
                kall[j * D + d] = load_elem(K, dtype, (j * H + h) * D + d);
                vall[j * D + d] = load_elem(V, dtype, (j * H + h) * D + d);
            }
        memset(dkall, 0, sizeof(double) * tok_elems * (size_t)nt);
        memset(dvall, 0, sizeof(double) * tok_elems * (size_t)nt);
        memset(dKc, 0, sizeof(double) * blk_elems * (size_t)nt);
        memset(dVc, 0, sizeof(double) * blk_elems * (size_t)nt);

#pragma omp parallel
        {
            const int t = omp_get_thread_num();
            double* my_dk = dkall + (size_t)t * tok_elems;
            double* my_dv = dvall + (size_t)t * tok_elems;
            double* my_dKc = dKc + (size_t)t * blk_elems;
            double* my_dVc = dVc + (size_t)t * blk_elems;
            double* q = (double*)malloc(sizeof(double) * (size_t)D);
            double* go = (double*)malloc(sizeof(double) * (size_t)D);
            double* dq = (double*)malloc(sizeof(double) * (size_t)D);
            double* P = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1));
            double* dP = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1));
            const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(max_keys + 1));
            const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(max_keys + 1));
            double** dkr = (double**)malloc(sizeof(double*) * (size_t)(max_keys + 1));
            double** dvr = (double**)malloc(sizeof(double*) * (size_t)(max_keys + 1));
#pragma omp for schedule(dynamic, 16)
            for (int64_t i = 0; i < n; ++i) {
                const float* g = &gates[(i * H + h) * 3];
                for (int32_t d = 0; d < D; ++d) {
                    q[d] = load_elem(Q, dtype, (i * H + h) * D + d);
                    go[d] = load_elem(dO, dtype, (i * H + h) * D + d);
                    dq[d] = 0.0;
                }
                /* compressed branch: keys Kc_b, values Vc_b */
                for (int64_t b = 0; b < mb; ++b) {
                    kr[b] = &Kc[(b * H + h) * D];
                    vr[b] = &Vc[(b * H + h) * D];
                    dkr[b] = &my_dKc[b * D];
                    dvr[b] = &my_dVc[b * D];
                }
                attend_backward(D, q, go, (double)g[0], mb, kr, vr, scale, P, dP, dq, dkr, dvr);
                /* selected branch */
                int64_t nk = 0;
                for (int32_t s = 0; s < topk; ++s) {
                    int32_t b = sel[(i * H + h) * topk + s];
                    if (b < 0) continue;
                    for (int64_t p = blk_off[b]; p < blk_off[b + 1]; ++p) {
                        int64_t j = perm[p];
                        kr[nk] = &kall[j * D];
                        vr[nk] = &vall[j * D];
                        dkr[nk] = &my_dk[j * D];
                        dvr[nk] = &my_dv[j * D];
                        nk += 1;
                    }
                }
                attend_backward(D, q, go, (double)g[1], nk, kr, vr, scale, P, dP, dq, dkr, dvr);
                /* window branch */
                nk = 0;
                for (int64_t tt = nbr_off[i]; tt < nbr_off[i + 1]; ++tt) {
                    int64_t j = nbr_idx[tt];
                    kr[nk] = &kall[j * D];
                    vr[nk] = &vall[j * D];
                    dkr[nk] = &my_dk[j * D];
                    dvr[nk] = &my_dv[j * D];
                    nk += 1;
                }
                attend_backward(D, q, go, (double)g[2], nk, kr, vr, scale, P, dP, dq, dkr, dvr);
                for (int32_t d = 0; d < D; ++d) dQ[(i * H + h) * D + d] = dq[d];
            }
            free(q); free(go); free(dq); free(P); free(dP); free(kr); free(vr); free(dkr); free(dvr);
        }

        /* the threads' partial key / value gradients, summed in thread order into copy 0 */
#pragma omp parallel for schedule(static)
        for (int64_t e = 0; e < n * D; ++e) {
            double sk = 0.0, sv = 0.0;
            for (int t = 0; t < nt; ++t) {
                sk += dkall[(size_t)t * tok_elems + (size_t)e];
                sv += dvall[(size_t)t * tok_elems + (size_t)e];
            }
            dkall[e] = sk;
            dvall[e] = sv;
        }
        for (int64_t e = 0; e < mb * D; ++e) {
            double sk = 0.0, sv = 0.0;
            for (int t = 0; t < nt; ++t) {
                sk += dKc[(size_t)t * blk_elems + (size_t)e];
                sv += dVc[(size_t)t * blk_elems + (size_t)e];
            }
            dKc[e] = sk;
            dVc[e] = sv;
        }

        /* through the compression: Kc_b = mean(K_b) . Wc  =>  dK_j += (1/n_b) dKc_b . Wc^T */
        for (int64_t b = 0; b < mb; ++b) {
            double inv = 1.0 / (double)(blk_off[b + 1] - blk_off[b]);
            for (int32_t d = 0; d < D; ++d) {
                double gk = 0.0, gv = 0.0;
                for (int32_t e = 0; e < D; ++e) {
                    gk += dKc[b * D + e] * (double)Wc[d * D + e];
                    gv += dVc[b * D + e] * (double)Wc[d * D + e];
                }
                for (int64_t p = blk_off[b]; p < blk_off[b + 1]; ++p) {
                    int64_t j = perm[p];
                    dkall[j * D + d] += inv * gk;
                    dvall[j * D + d] += inv * gv;
                }
            }
        }
        for (int64_t j = 0; j < n; ++j)
            for (int32_t d = 0; d < D; ++d) {
                dK[(j * H + h) * D + d] = dkall[j * D + d];
                dV[(j * H + h) * D + d] = dvall[j * D + d];
            }
    }
    free(kall); free(vall); free(dkall); free(dvall); free(dKc); free(dVc);
    free(Kc);
    free(Vc);
    return 0;
}

/*
 * dQ only, for a set of rows: dQ_i needs nothing but row i's own forward quantities, so it
 * can be evaluated at any size. Same conventions as oracle_backward; dQ is [n_rows, H, D].
 * sel_in ([n_rows, H, k] local block indices) replaces the computed selection when non-NULL;
 * sel_out receives the selection used.
 */
int oracle_backward_dq_rows(int64_t n, int32_t H, int32_t D, int32_t dtype, const void* Q,
                            const void* K, const void* V, const float* gates, const float* Wc,
                            const void* dO, int32_t topk, int32_t round_compressed,
                            const int32_t* perm, const int32_t* tok_blk, const int32_t* blk_off,
                            int64_t mb, const int64_t* nbr_off, const int32_t* nbr_idx,
                            int64_t n_rows, const int64_t* rows, const int32_t* sel_in,
                            double* dQ, int32_t* sel_out) {
    double* Kc = (double*)malloc(sizeof(double) * (size_t)(mb * H * D + 1));
    double* Vc = (double*)malloc(sizeof(double) * (size_t)(mb * H * D + 1));
    if (!Kc || !Vc) return -1;
    compress(mb, H, D, dtype, K, V, Wc, perm, blk_off, round_compressed, Kc, Vc);
    const double scale = 1.0 / sqrt((double)D);
    int64_t max_nb = 0;
    for (int64_t b = 0; b < mb; ++b)
        if (blk_off[b + 1] - blk_off[b] > max_nb) max_nb = blk_off[b + 1] - blk_off[b];
    int64_t max_keys = max_nb * topk;
    for (int64_t i = 0; i < n; ++i)
        if (nbr_off[i + 1] - nbr_off[i] > max_keys) max_keys = nbr_off[i + 1] - nbr_off[i];
    if (mb > max_keys) max_keys = mb;
#pragma omp parallel
    {
        double* q = (double*)malloc(sizeof(double) * (size_t)D);
        double* go = (double*)malloc(sizeof(double) * (size_t)D);
        double* dq = (double*)malloc(sizeof(double) * (size_t)D);
        double* z = (double*)malloc(sizeof(double) * (size_t)(mb + 1));
        int32_t* s_loc = (int32_t*)malloc(sizeof(int32_t) * (size_t)topk);
        double* P = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1));
        double* dP = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1));
        double* kbuf = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1) * (size_t)D);
        double* vbuf = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1) * (size_t)D);
        const double** kr = (const double**)malloc(sizeof(double*) * (size_t)(max_keys + 1));
        const double** vr = (const double**)malloc(sizeof(double*) * (size_t)(max_keys + 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t rh = 0; rh < n_rows * H; ++rh) {
            int64_t ri = rh / H;
            int32_t h = (int32_t)(rh % H);
            int64_t i = rows[ri];
            const float* g = &gates[(i * H + h) * 3];
            for (int32_t d = 0; d < D; ++d) {
                q[d] = load_elem(Q, dtype, (i * H + h) * D + d);
                go[d] = load_elem(dO, dtype, (i * H + h) * D + d);
                dq[d] = 0.0;
            }
            for (int64_t b = 0; b < mb; ++b) {
                double t = 0.0;
                for (int32_t d = 0; d < D; ++d) t += q[d] * Kc[(b * H + h) * D + d];
                z[b] = scale * t;
                kr[b] = &Kc[(b * H + h) * D];
                vr[b] = &Vc[(b * H + h) * D];
            }
            attend_backward(D, q, go, (double)g[0], mb, kr, vr, scale, P, dP, dq, NULL, NULL);
            if (sel_in) {
                for (int32_t s = 0; s < topk; ++s) s_loc[s] = sel_in[(ri * H + h) * topk + s];
            } else {
                select_blocks(mb, z, tok_blk[i], topk, s_loc);
            }
            if (sel_out)
                for (int32_t s = 0; s < topk; ++s) sel_out[(ri * H + h) * topk + s] = s_loc[s];
            int64_t nk = 0;
            for (int32_t s = 0; s < topk; ++s) {
                int32_t b = s_loc[s];
                if (b < 0) continue;
                for (int64_t p = blk_off[b]; p < blk_off[b + 1]; ++p) {
                    int64_t j = perm[p];
                    for (int32_t d = 0; d < D; ++d) {
                        kbuf[nk * D + d] = load_elem(K, dtype, (j * H + h) * D + d);
                        vbuf[nk * D + d] = load_elem(V, dtype, (j * H + h) * D + d);
                    }
                    kr[nk] = &kbuf[nk * D];
                    vr[nk] = &vbuf[nk * D];
                    nk += 1;
                }
            }
            attend_backward(D, q, go, (double)g[1], nk, kr, vr, scale, P, dP, dq, NULL, NULL);
            nk = 0;
            for (int64_t t = nbr_off[i]; t < nbr_off[i + 1]; ++t) {
                int64_t j = nbr_idx[t];
                for (int32_t d = 0; d < D; ++d) {
                    kbuf[nk * D + d] = load_elem(K, dtype, (j * H + h) * D + d);
                    vbuf[nk * D + d] = load_elem(V, dtype, (j * H + h) * D + d);
                }
                kr[nk] = &kbuf[nk * D];
                vr[nk] = &vbuf[nk * D];
                nk += 1;
            }
            attend_backward(D, q, go, (double)g[2], nk, kr, vr, scale, P, dP, dq, NULL, NULL);
            for (int32_t d = 0; d < D; ++d) dQ[(ri * H + h) * D + d] = dq[d];
        }
        free(q); free(go); free(dq); free(z); free(s_loc); free(P); free(dP);
        free(kbuf); free(vbuf); free(kr); free(vr);
    }
    free(Kc);
    free(Vc);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* 9. attention prologue: RMS normalisation of queries and keys, 3D rotary position embedding  */
/* ------------------------------------------------------------------------------------------ */

/*
 * Hi3D v1.0 pipeline page, "Stage 3: sparse flow sampling": the transformer that runs attention
 * over the sparse voxel tokens applies rotary position embeddings and RMS normalisation to the
 * self-attention queries and keys. The page gives no formulas; this is the plain reading:
 *   1. RMS normalisation over the head dimension, one weight vector per operand (gamma, length
 *      D) shared by all heads: u_d = x_d / sqrt(mean_e x_e^2 + eps) * gamma_d;
 *   2. 3D rotary embedding with the token's voxel coordinates as positions: the head dimension
 *      is cut into an x part, a y part and a z part (oracle_rope_split), and channel pair
 *      (c, c+1) of the part for axis a, j-th pair of that part, is rotated by the angle
 *      coords[a] * theta^(-2j / width_a):  (u, v) -> (u cos t - v sin t, u sin t + v cos t).
 * Like any layer of the model, the prologue hands its queries and keys on in the input type:
 * the method runs on the results rounded to it (oracle_round_array, applied by the caller).
 */

/* Widths of the x, y and z parts: y and z get 2*floor(D/6) channels each, x the rest. */
void oracle_rope_split(int32_t D, int32_t* wx, int32_t* wy, int32_t* wz) {
    int32_t c = 2 * (D / 6);
    *wy = c;
    *wz = c;
    *wx = D - 2 * c;
}

/* out[n, H, D] (double) = rotary(rmsnorm(X)) for every token and head; X of `dtype`. */
int oracle_qk_prologue(int64_t n, int32_t H, int32_t D, int32_t dtype, const void* X,
                       const int32_t* coords, const float* gamma, double eps, double theta,
                       double* out) {
    if (D < 2 || (D & 1) || H < 1) return -1;
    int32_t w[3];
    oracle_rope_split(D, &w[0], &w[1], &w[2]);
#pragma omp parallel for schedule(static)
    for (int64_t ih = 0; ih < n * H; ++ih) {
        int64_t i = ih / H;
        double* o = out + ih * D;
        double ss = 0.0;
        for (int32_t d = 0; d < D; ++d) {
            o[d] = load_elem(X, dtype, ih * D + d);
            ss += o[d] * o[d];
        }
        double inv = 1.0 / sqrt(ss / (double)D + eps);
        for (int32_t d = 0; d < D; ++d) o[d] = o[d] * inv * (double)gamma[d];
        int32_t start = 0;
        for (int32_t a = 0; a < 3; ++a) {
            double pos = (double)coords[3 * i + a];
            for (int32_t j = 0; j < w[a] / 2; ++j) {
                double t = pos * pow(theta, -2.0 * (double)j / (double)w[a]);
                double u = o[start + 2 * j], v = o[start + 2 * j + 1];
                o[start + 2 * j] = u * cos(t) - v * sin(t);
                o[start + 2 * j + 1] = u * sin(t) + v * cos(t);
            }
            start += w[a];
        }
    }
    return 0;
}

/* x[0..n) rounded in place to the storage type `dtype` (oracle_round_to, element by element). */
void oracle_round_array(double* x, int64_t n, int32_t dtype) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) x[i] = oracle_round_to(x[i], dtype);
}
