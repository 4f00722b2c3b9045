/*
 * nl_oracle.c -- CPU oracle for the periodic neighbor-list build.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow restatement of what
 * the neighbor-list hot path computes.  Only the test suite, the smoke
 * check and the benchmark's CPU-baseline / reference leg may load it.  The
 * product library never calls, links or includes it, and the two share no
 * code, headers or constants.
 *
 * Source of the method: "Ab Initio Accuracy Beyond the Cutoff: Distributed
 * Message-Passing Equivariant Attention at Tens-of-Millions-of-Atom Scale"
 * (Tessera), abstract:
 *   - atoms are sorted along a space-filling curve (contrasted there with
 *     Morton order; the curve used here is the 3-D Hilbert curve);
 *   - a conservative neighbor skin keeps the neighbor topology fixed between
 *     rebuilds, so tensor shapes stay fixed (fixed-capacity padded rows);
 *   - a skin check decides when a rebuild is needed.
 * The pages print no formulas for these steps.  The readings taken here:
 *   wrap        w = x - L*floor(x/L), then one correction into [0, L)
 *   quantize    q = min(floor(w * fl(2^21 / L)), 2^21 - 1)
 *   Hilbert     J. Skilling, "Programming the Hilbert curve", AIP Conf. Proc.
 *               707 (2004): the axes-to-transpose transform, index bits read
 *               from the top level down, axis 0 first in each triple
 *   order       sort of (key, original index) pairs
 *   distance    d = wj - wi;  d = d - L*rintf(d/L);  r2 = (dx*dx+dy*dy)+dz*dz
 *               in fp32 round-to-nearest, no fused multiply-add
 *   neighbors   j != i with r2 < rl2, rl = fl(cutoff+skin), rl2 = fl(rl*rl)
 *   rows        ascending, first K kept, rest -1, counts = true count
 *   skin check  max_i r2(x_i - ref_i) > fl(h*h), h = fl(skin*0.5)
 * Every function below computes its definition directly; the cell list only
 * enumerates candidates, the predicate decides.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp (x86-64 SSE
 * arithmetic).  Three loops run on OpenMP threads, each over independent
 * elements: the keys of the atoms, their wrapped coordinates, and the rows
 * of oracle_rows (each row computed and sorted by one thread).  No result
 * depends on the thread count; oracle_set_threads(1) makes the oracle
 * single-threaded.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_QBITS 21
#define OR_QMAX ((1u << OR_QBITS) - 1u)

/* ------------------------------------------------------------------ wrap */

/* Periodic wrap of one coordinate into [0, L) (reading of "periodic box";
 * the pages give no formula).  Each operation is one fp32 rounding. */
float oracle_wrap(float x, float L)
{
    float t = floorf(x / L);
    float lt = L * t;
    float w = x - lt;
    if (w < 0.0f) w = w + L;
    if (w >= L) w = w - L;
    if (!(w >= 0.0f && w < L)) w = 0.0f;
    return w;
}

/* 21-bit grid coordinate of a wrapped coordinate; S = fl(2^21 / L). */
uint32_t oracle_quantize(float w, float S)
{
    float v = w * S;
    float f = floorf(v);
    uint32_t q;
    if (!(f >= 0.0f)) return 0u;
    if (f >= 2097152.0f) return OR_QMAX;
    q = (uint32_t)f;
    return q > OR_QMAX ? OR_QMAX : q;
}

float oracle_quant_scale(float L)
{
    return 2097152.0f / L;
}

/* ------------------------------------------------------------- Hilbert */

/* Skilling (2004), axes -> transposed Hilbert index, n = 3 dimensions,
 * b bits per axis.  Written as that paper states the transform: undo the
 * excess work of the inverse, then Gray-encode. */
static void or_axes_to_transpose(uint32_t X[3], int b)
{
    uint32_t M = 1u << (b - 1);
    uint32_t Q, P, t;
    int i;
    for (Q = M; Q > 1; Q >>= 1) {
        P = Q - 1;
        for (i = 0; i < 3; i++) {
            if (X[i] & Q) {
                X[0] ^= P;                 /* invert low bits of X[0] */
            } else {
                t = (X[0] ^ X[i]) & P;     /* exchange low bits */
                X[0] ^= t;
                X[i] ^= t;
            }
        }
    }
    for (i = 1; i < 3; i++) X[i] ^= X[i - 1];
    t = 0;
    for (Q = M; Q > 1; Q >>= 1)
        if (X[2] & Q) t ^= Q - 1;
    for (i = 0; i < 3; i++) X[i] ^= t;
}

/* Skilling (2004), transposed Hilbert index -> axes (the inverse). */
static void or_transpose_to_axes(uint32_t X[3], int b)
{
    uint32_t N = 2u << (b - 1);
    uint32_t Q, P, t;
    int i;
    t = X[2] >> 1;
    for (i = 2; i > 0; i--) X[i] ^= X[i - 1];
    X[0] ^= t;
    for (Q = 2; Q != N; Q <<= 1) {
        P = Q - 1;
        for (i = 2; i >= 0; i--) {
            if (X[i] & Q) {
                X[0] ^= P;
            } else {
                t = (X[0] ^ X[i]) & P;
                X[0] ^= t;
                X[i] ^= t;
            }
        }
    }
}

/* Hilbert index of grid cell (qx, qy, qz) on a 2^b grid: the transposed
 * digits read from level b-1 down to 0, axis 0 first in each triple. */
uint64_t oracle_hilbert_key(uint32_t qx, uint32_t qy, uint32_t qz, int b)
{
    uint32_t X[3];
    uint64_t key = 0;
    int l, d;
    X[0] = qx; X[1] = qy; X[2] = qz;
    or_axes_to_transpose(X, b);
    for (l = b - 1; l >= 0; l--)
        for (d = 0; d < 3; d++)
            key = (key << 1) | (uint64_t)((X[d] >> l) & 1u);
    return key;
}

/* Grid cell of Hilbert index `key` on a 2^b grid (inverse of the above). */
void oracle_hilbert_axes(uint64_t key, int b, uint32_t out[3])
{
    uint32_t X[3] = {0u, 0u, 0u};
    int l, d, pos = 3 * b - 1;
    for (l = b - 1; l >= 0; l--)
        for (d = 0; d < 3; d++) {
            X[d] |= (uint32_t)((key >> pos) & 1u) << l;
            pos--;
        }
    or_transpose_to_axes(X, b);
    out[0] = X[0]; out[1] = X[1]; out[2] = X[2];
}

/* Morton (Z-order) index: bit 3l+2 = x_l, 3l+1 = y_l, 3l = z_l. */
uint64_t oracle_morton_key(uint32_t qx, uint32_t qy, uint32_t qz, int b)
{
    uint64_t key = 0;
    int l;
    for (l = b - 1; l >= 0; l--) {
        key = (key << 1) | ((qx >> l) & 1u);
        key = (key << 1) | ((qy >> l) & 1u);
        key = (key << 1) | ((qz >> l) & 1u);
    }
    return key;
}

/* Keys of all atoms.  pos4: n x 4 floats (x, y, z, ignored).  curve 0 =
 * Hilbert, 1 = Morton. */
void oracle_keys(int64_t n, const float *pos4, const float box[3], int curve,
                 uint64_t *keys)
{
    float S[3];
    int64_t i;
    int a;
    for (a = 0; a < 3; a++) S[a] = oracle_quant_scale(box[a]);
#pragma omp parallel for private(a) schedule(static)
    for (i = 0; i < n; i++) {
        uint32_t q[3];
        for (a = 0; a < 3; a++)
            q[a] = oracle_quantize(oracle_wrap(pos4[4 * i + a], box[a]), S[a]);
        keys[i] = curve == 1 ? oracle_morton_key(q[0], q[1], q[2], OR_QBITS)
                             : oracle_hilbert_key(q[0], q[1], q[2], OR_QBITS);
    }
}

typedef struct {
    uint64_t key;
    int64_t idx;
} or_pair;

static int or_cmp_pair(const void *a, const void *b)
{
    const or_pair *p = (const or_pair *)a, *q = (const or_pair *)b;
    if (p->key != q->key) return p->key < q->key ? -1 : 1;
    if (p->idx != q->idx) return p->idx < q->idx ? -1 : 1;
    return 0;
}

/* Curve order: perm[k] = index of the k-th (key, index) pair in ascending
 * order, i.e. a stable sort by key.  keys_sorted may be NULL. */
int oracle_sort(int64_t n, const float *pos4, const float box[3], int curve,
                int32_t *perm, uint64_t *keys_sorted)
{
    uint64_t *keys;
    or_pair *pairs;
    int64_t i;
    if (n <= 0) return 0;
    keys = (uint64_t *)malloc((size_t)n * sizeof(uint64_t));
    pairs = (or_pair *)malloc((size_t)n * sizeof(or_pair));
    if (!keys || !pairs) { free(keys); free(pairs); return -1; }
    oracle_keys(n, pos4, box, curve, keys);
    for (i = 0; i < n; i++) { pairs[i].key = keys[i]; pairs[i].idx = i; }
    qsort(pairs, (size_t)n, sizeof(or_pair), or_cmp_pair);
    for (i = 0; i < n; i++) {
        perm[i] = (int32_t)pairs[i].idx;
        if (keys_sorted) keys_sorted[i] = pairs[i].key;
    }
    free(keys);
    free(pairs);
    return 0;
}

/* ------------------------------------------------------------ distance */

/* Minimum image of one component: d - L*rintf(d/L). */
float oracle_min_image(float d, float L)
{
    float r = rintf(d / L);
    float lr = L * r;
    return d - lr;
}

/* Squared minimum-image distance between two points, (dx*dx+dy*dy)+dz*dz. */
float oracle_r2(const float a[3], const float b[3], const float box[3])
{
    float dx = oracle_min_image(b[0] - a[0], box[0]);
    float dy = oracle_min_image(b[1] - a[1], box[1]);
    float dz = oracle_min_image(b[2] - a[2], box[2]);
    float xx = dx * dx, yy = dy * dy, zz = dz * dz;
    float s = xx + yy;
    return s + zz;
}

/* ----------------------------------------------------- neighbor lists */

typedef struct {
    int32_t *v;
    int64_t n, cap;
} or_vec;

static int or_push(or_vec *v, int32_t x)
{
    if (v->n == v->cap) {
        int64_t c = v->cap ? 2 * v->cap : 256;
        int32_t *p = (int32_t *)realloc(v->v, (size_t)c * sizeof(int32_t));
        if (!p) return -1;
        v->v = p;
        v->cap = c;
    }
    v->v[v->n++] = x;
    return 0;
}

static int or_cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Writes one padded row from an unsorted hit list; returns 1 on overflow. */
static int or_emit_row(or_vec *hits, int32_t K, int32_t *row, int32_t *count)
{
    int64_t k;
    qsort(hits->v, (size_t)hits->n, sizeof(int32_t), or_cmp_i32);
    for (k = 0; k < K; k++) row[k] = k < hits->n ? hits->v[k] : -1;
    *count = (int32_t)hits->n;
    return hits->n > K;
}

static float *or_wrap_all(int64_t n, const float *pos4, const float box[3])
{
    float *w = (float *)malloc((size_t)(n > 0 ? n : 1) * 3 * sizeof(float));
    int64_t i;
    int a;
    if (!w) return NULL;
#pragma omp parallel for private(a) schedule(static)
    for (i = 0; i < n; i++)
        for (a = 0; a < 3; a++) w[3 * i + a] = oracle_wrap(pos4[4 * i + a], box[a]);
    return w;
}

/* O(N^2) definition: for every i, every j != i in index order. */
int oracle_bruteforce(int64_t n, const float *pos4, const float box[3],
                      float cutoff, float skin, int32_t K, int32_t *nbr,
                      int32_t *counts)
{
    float rl = cutoff + skin;
    float rl2 = rl * rl;
    float *w = or_wrap_all(n, pos4, box);
    or_vec hits = {0, 0, 0};
    int64_t i, j;
    int over = 0;
    if (!w) return -1;
    for (i = 0; i < n; i++) {
        hits.n = 0;
        for (j = 0; j < n; j++) {
            if (j == i) continue;
            if (oracle_r2(&w[3 * i], &w[3 * j], box) < rl2)
                if (or_push(&hits, (int32_t)j)) { free(w); free(hits.v); return -1; }
        }
        over |= or_emit_row(&hits, K, nbr + i * (int64_t)K, counts + i);
    }
    free(w);
    free(hits.v);
    return over;
}

/* Rows of the neighbor list for the atoms listed in `rows` (all atoms when
 * rows == NULL, nrows = n).  Candidates come from a linked-cell list whose
 * cells are at least rl*(1 + 1e-4) wide, assigned in double precision; every
 * candidate is then tested with the fp32 predicate above.  Boxes narrower
 * than three such cells fall back to testing every atom.
 * Returns 1 if any listed row has more than K neighbors, 0 otherwise. */
int oracle_rows(int64_t n, const float *pos4, const float box[3], float cutoff,
                float skin, int32_t K, int64_t nrows, const int64_t *rows,
                int32_t *nbr, int32_t *counts)
{
    float rl = cutoff + skin;
    float rl2 = rl * rl;
    int m[3], a, over = 0, brute = 0;
    volatile int failed = 0;
    int64_t ncell = 1, r, i;
    int64_t *head = NULL, *next = NULL, *cellof = NULL;
    float *w;

    w = or_wrap_all(n, pos4, box);
    if (!w) return -1;
    for (a = 0; a < 3; a++) {
        double side = (double)rl * (1.0 + 1e-4);
        double mm = floor((double)box[a] / side);
        m[a] = mm > 1024.0 ? 1024 : (int)mm;
        if (m[a] < 3) brute = 1;
        ncell *= m[a] > 0 ? m[a] : 1;
    }
    if (!brute) {
        head = (int64_t *)malloc((size_t)ncell * sizeof(int64_t));
        next = (int64_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof(int64_t));
        cellof = (int64_t *)malloc((size_t)(n > 0 ? n : 1) * 3 * sizeof(int64_t));
        if (!head || !next || !cellof) { brute = 1; }
    }
    if (!brute) {
        for (r = 0; r < ncell; r++) head[r] = -1;
        for (i = n - 1; i >= 0; i--) {
            int64_t c[3], id;
            for (a = 0; a < 3; a++) {
                double u = floor((double)w[3 * i + a] / (double)box[a] * (double)m[a]);
                if (u < 0) u = 0;
                if (u > m[a] - 1) u = m[a] - 1;
                c[a] = (int64_t)u;
                cellof[3 * i + a] = c[a];
            }
            id = (c[2] * m[1] + c[1]) * m[0] + c[0];
            next[i] = head[id];
            head[id] = i;
        }
    }
    /* Rows are independent and each is sorted before it is written, so the
     * result does not depend on how the rows are shared out among threads. */
#pragma omp parallel reduction(| : over)
    {
        or_vec hits = {0, 0, 0};
        int64_t rr;
#pragma omp for schedule(dynamic, 256)
        for (rr = 0; rr < nrows; rr++) {
            int64_t ii = rows ? rows[rr] : rr, jj;
            if (failed) continue;
            hits.n = 0;
            if (brute) {
                for (jj = 0; jj < n; jj++)
                    if (jj != ii && oracle_r2(&w[3 * ii], &w[3 * jj], box) < rl2)
                        if (or_push(&hits, (int32_t)jj)) { failed = 1; break; }
            } else {
                int ox, oy, oz;
                for (oz = -1; oz <= 1; oz++)
                    for (oy = -1; oy <= 1; oy++)
                        for (ox = -1; ox <= 1; ox++) {
                            int64_t cx = (cellof[3 * ii + 0] + ox + m[0]) % m[0];
                            int64_t cy = (cellof[3 * ii + 1] + oy + m[1]) % m[1];
                            int64_t cz = (cellof[3 * ii + 2] + oz + m[2]) % m[2];
                            for (jj = head[(cz * m[1] + cy) * m[0] + cx]; jj >= 0; jj = next[jj])
                                if (jj != ii && oracle_r2(&w[3 * ii], &w[3 * jj], box) < rl2)
                                    if (or_push(&hits, (int32_t)jj)) failed = 1;
                        }
            }
            if (!failed) over |= or_emit_row(&hits, K, nbr + rr * (int64_t)K, counts + rr);
        }
        free(hits.v);
    }
    free(w); free(head); free(next); free(cellof);
    return failed ? -1 : over;
}

/* Number of threads the row loops of the oracle may use (OpenMP); 1 gives
 * the plain single-threaded oracle.  Returns the previous setting. */
int oracle_set_threads(int nthreads)
{
#ifdef _OPENMP
    int old = omp_get_max_threads();
    if (nthreads >= 1) omp_set_num_threads(nthreads);
    return old;
#else
    (void)nthreads;
    return 1;
#endif
}

int oracle_build(int64_t n, const float *pos4, const float box[3], float cutoff,
                 float skin, int32_t K, int32_t *nbr, int32_t *counts)
{
    return oracle_rows(n, pos4, box, cutoff, skin, K, n, NULL, nbr, counts);
}

/* Close-pair detector over the full neighbor sets (no capacity cut): the
 * smallest r2 of any directed neighbor pair (i, j in N(i)), +inf when there
 * is none, and the number of directed neighbor pairs with r2 < close_d2.
 * Reading of the pages' "no anomalously close pairs" check (Tessera,
 * abstract): a by-product of the same predicate and candidate set.
 * Returns 0, or -1 when memory runs out. */
int oracle_close_pairs(int64_t n, const float *pos4, const float box[3], float cutoff,
                       float skin, float close_d2, float *min_d2, int64_t *n_close)
{
    int32_t *cnt = (int32_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof(int32_t));
    int32_t *one = (int32_t *)malloc((size_t)(n > 0 ? n : 1) * sizeof(int32_t));
    int32_t *nbr = NULL, K = 1;
    float *w = NULL, mn = INFINITY;
    int64_t i, k, nc = 0;
    if (!cnt || !one) goto fail;
    if (oracle_rows(n, pos4, box, cutoff, skin, 1, n, NULL, one, cnt) < 0) goto fail;
    for (i = 0; i < n; i++)
        if (cnt[i] > K) K = cnt[i];
    nbr = (int32_t *)malloc((size_t)(n > 0 ? n : 1) * (size_t)K * sizeof(int32_t));
    if (!nbr) goto fail;
    if (oracle_rows(n, pos4, box, cutoff, skin, K, n, NULL, nbr, cnt) < 0) goto fail;
    w = or_wrap_all(n, pos4, box);
    if (!w) goto fail;
    for (i = 0; i < n; i++)
        for (k = 0; k < cnt[i]; k++) {
            int64_t j = nbr[i * (int64_t)K + k];
            float r2 = oracle_r2(&w[3 * i], &w[3 * j], box);
            if (r2 < mn) mn = r2;
            if (r2 < close_d2) nc++;
        }
    *min_d2 = mn;
    *n_close = nc;
    free(cnt); free(one); free(nbr); free(w);
    return 0;
fail:
    free(cnt); free(one); free(nbr); free(w);
    return -1;
}

/* --------------------------------------------------------- edge features */

/* Per-slot edge features of padded rows (reading of the pages' padded,
 * dense neighbor tensors that the message-passing layers consume; Tessera,
 * abstract, and the page on batching and kernel fusion): for row i and slot
 * s < min(counts[i], K), j = nbr[i][s] and
 *     (dx, dy, dz) = minimum image of w_j - w_i, per axis as in oracle_r2,
 *     r = sqrtf((dx*dx + dy*dy) + dz*dz)   (IEEE square root, one rounding),
 * written as out[(i*K + s)*4 + 0..3]; every other slot is (0, 0, 0, 0).
 * An index outside [0, n) also gives zeros.  The rows may come from any
 * builder: the features depend only on (i, j). */
void oracle_edge_features(int64_t n, const float *pos4, const float box[3], int32_t K,
                          const int32_t *nbr, const int32_t *counts, float *out)
{
    int64_t i, s;
    for (i = 0; i < n; i++) {
        float wi[3], wj[3];
        int32_t c = counts[i] < K ? counts[i] : K;
        int a;
        for (a = 0; a < 3; a++) wi[a] = oracle_wrap(pos4[4 * i + a], box[a]);
        for (s = 0; s < K; s++) {
            float *o = out + 4 * (i * (int64_t)K + s);
            int64_t j = s < c ? nbr[i * (int64_t)K + s] : -1;
            o[0] = o[1] = o[2] = o[3] = 0.0f;
            if (j < 0 || j >= n) continue;
            for (a = 0; a < 3; a++) wj[a] = oracle_wrap(pos4[4 * j + a], box[a]);
            {
                float dx = oracle_min_image(wj[0] - wi[0], box[0]);
                float dy = oracle_min_image(wj[1] - wi[1], box[1]);
                float dz = oracle_min_image(wj[2] - wi[2], box[2]);
                float r2 = oracle_r2(wi, wj, box);
                o[0] = dx;
                o[1] = dy;
                o[2] = dz;
                o[3] = sqrtf(r2);
            }
        }
    }
}

/* ----------------------------------------------------------- skin check */

/* Largest squared minimum-image displacement since the reference positions,
 * on the raw (unwrapped) coordinates; *rebuild = (max > fl(h*h)). */
float oracle_skin_check(int64_t n, const float *pos4, const float *ref4,
                        const float box[3], float skin, int32_t *rebuild)
{
    float h = skin * 0.5f;
    float h2 = h * h;
    float m = 0.0f;
    int64_t i;
    for (i = 0; i < n; i++) {
        float a[3], b[3];
        float r2;
        int c;
        for (c = 0; c < 3; c++) { a[c] = ref4[4 * i + c]; b[c] = pos4[4 * i + c]; }
        r2 = oracle_r2(a, b, box);
        if (r2 > m) m = r2;
    }
    if (rebuild) *rebuild = m > h2 ? 1 : 0;
    return m;
}

/* ----------------------------------------- synthetic dynamics stand-in */

/* SplitMix64 (Steele, Lea & Flood, OOPSLA 2014; constants as published by
 * Vigna): one output for one 64-bit counter. */
static uint64_t or_splitmix64(uint64_t x)
{
    uint64_t z = x + 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

/* Displacement of atom `atom` along `axis` at MD step `step` (>= 1): the sum
 * of the four 16-bit fields of one SplitMix64 output, centred (an
 * Irwin-Hall(4) variate, exact in integers), times
 * A = fl(sigma * sqrt(3) / 65536), so its standard deviation is sigma. */
float oracle_displacement(uint64_t seed, int64_t step, int64_t atom, int axis,
                          float sigma)
{
    uint64_t ctr = ((uint64_t)step << 42) | ((uint64_t)atom << 2) | (uint64_t)axis;
    uint64_t u = or_splitmix64(or_splitmix64(seed) + ctr);
    int32_t s = (int32_t)(u & 0xffffu) + (int32_t)((u >> 16) & 0xffffu) +
                (int32_t)((u >> 32) & 0xffffu) + (int32_t)((u >> 48) & 0xffffu);
    float g = (float)(s - 131070);
    float A = (float)((double)sigma * sqrt(3.0) / 65536.0);
    return g * A;
}

/* x <- fl(x + delta(step)) for every atom and axis. */
void oracle_displace(int64_t n, float *pos4, uint64_t seed, int64_t step, float sigma)
{
    int64_t i;
    int a;
    for (i = 0; i < n; i++)
        for (a = 0; a < 3; a++)
            pos4[4 * i + a] = pos4[4 * i + a] + oracle_displacement(seed, step, i, a, sigma);
}

/* Skin-check loop: ref = pos at entry (the step-0 build); for t = 1..T the
 * positions move by delta(t), the check runs, and a rebuild (ref <- pos) is
 * recorded in decisions[t-1].  pos4 and ref4 are updated in place; returns
 * the number of rebuilds. */
int64_t oracle_md_decisions(int64_t n, float *pos4, float *ref4, const float box[3],
                            float skin, uint64_t seed, float sigma, int64_t steps,
                            int32_t *decisions)
{
    int64_t t, rebuilds = 0;
    memcpy(ref4, pos4, (size_t)n * 4 * sizeof(float));
    for (t = 1; t <= steps; t++) {
        int32_t rb = 0;
        oracle_displace(n, pos4, seed, t, sigma);
        oracle_skin_check(n, pos4, ref4, box, skin, &rb);
        decisions[t - 1] = rb;
        if (rb) {
            memcpy(ref4, pos4, (size_t)n * 4 * sizeof(float));
            rebuilds++;
        }
    }
    return rebuilds;
}
