/*
 * attention_oracle.c -- TEST INFRASTRUCTURE, NOT PRODUCT CODE.
 *
 * A plain, slow, fp64 CPU implementation of exact scaled-dot-product
 * attention (forward and backward, optional causal mask, optional dropout).
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this library.  It shares no code, header, table or constant
 * generator with the CUDA library it checks; the CUDA library never loads it.
 *
 * What it computes (every quantity in double precision; inputs are either
 * bf16 bit patterns, widened exactly to double, or doubles -- the latter only
 * for the finite-difference pins):
 *
 *   s_ij  = scale * <q_i, k_j>            ; -inf where causal and j > i
 *   m_i   = max_j s_ij                     (two-pass, NOT online)
 *   l_i   = sum_j exp(s_ij - m_i)
 *   P_ij  = exp(s_ij - m_i) / l_i
 *   lse_i = m_i + ln(l_i)
 *   Z_ij  = [h16(i,j) >= T]                ; T = ceil(p * 2^16), p=0 keeps all
 *   Pd_ij = P_ij * Z_ij / (1 - p)          (dropout applied after softmax)
 *   O_i   = sum_j Pd_ij v_j
 *
 * Backward, given dO (chain rule through the definition above):
 *   dV_j  = sum_i Pd_ij dO_i
 *   dP_ij = <dO_i, v_j> * Z_ij / (1 - p)
 *   D_i   = sum_j P_ij dP_ij               (equals <dO_i, O_i>; checked)
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 *
 * Sources:
 *  - definition softmax(QK^T/sqrt(d_k))V and the stable form exp(x - max):
 *    "FlashAttention for Efficient Training", section 1 (Basics of
 *    Self-Attention) and section 6.2 (numerically stable softmax equation);
 *  - the standard (unfused) order S -> P -> O, with S and P materialised:
 *    "How FlashAttention Optimizes GPU Memory for Fast AI Training",
 *    "The Flaw in Standard Attention";
 *  - causal masking inside the kernel: "FlashAttention for Efficient
 *    Training", section 5.1 (memory-efficient backward pass);
 *  - logsumexp statistic: same page, section 3.2 (log_softmax equation);
 *  - dV = P^T dO: same page, section 3.2 (Integration with Autograd Engines);
 *  - dropout fused after softmax scaling: same page, section 3 (Fused Kernel
 *    Design) and section 6.1 (Kernel Fusion Overhead);
 *  - block-sparse attention, only non-zero blocks of the attention matrix
 *    computed: same page, section 3.2 (Block-Sparse Attention Support).  An
 *    optional mask over tile x tile blocks hides keys (s_ij = -inf); a row
 *    that sees no key at all gets P = 0, O = 0 and lse = -inf (the pages do
 *    not say; this is the limit of an empty softmax taken as zero weight).
 *  - variable sequence lengths: "FlashAttention for Efficient Training",
 *    section 5.2 (Handling Variable Sequence Lengths, Efficient Padding and
 *    Masking: a score is -inf unless its key lies within the sequence,
 *    j <= L_i with 1-based j).  An optional per-batch length L_b makes the
 *    rows and keys at or beyond L_b of batch entry b padding: key j (0-based)
 *    is visible to query i iff j < L_b, and a padding query row i >= L_b has
 *    no keys at all (O = 0, lse = -inf, no gradient), so dK = dV = 0 for
 *    padding keys.  Padding values never enter any result.
 * The pages print garbled dQ formulas; the dQ/dK expressions here are the
 * chain rule, pinned by finite differences in the tests.
 *
 * Work is split over (head, row) pairs with OpenMP threads; every row is
 * computed independently from scratch, so the result does not depend on the
 * thread count.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- inputs */

static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    const void *q, *k, *v, *dout; /* [B,H,N,d]: bf16 bit patterns, or doubles if f64 */
    int f64;
    int B, H, N, d;
    double scale;
    int causal;
    double p_drop;
    uint64_t seed;
    /* optional block mask: bmask[hm][i / tile][j / tile] == 0 hides keys j from
     * queries i (hm = 0 if bmask_heads == 1, else the head h) */
    const uint8_t *bmask;
    int bmask_heads, bmask_tile;
    /* optional lengths [B]: rows/keys >= seqlens[b] of batch entry b are padding */
    const int32_t *seqlens;
} problem_t;

/* A row of one [B,H,N,d] input: base pointer plus its element type. */
typedef struct {
    const void *p;
    int f64;
} row_t;

static row_t row_ptr(const problem_t *pb, const void *t, int bh, int r) {
    size_t off = ((size_t)bh * pb->N + (size_t)r) * (size_t)pb->d;
    row_t rw;
    rw.f64 = pb->f64;
    rw.p = pb->f64 ? (const void *)((const double *)t + off) : (const void *)((const uint16_t *)t + off);
    return rw;
}

static double elem(row_t r, int c) {
    return r.f64 ? ((const double *)r.p)[c] : bf16_to_double(((const uint16_t *)r.p)[c]);
}

static double dot_rows(row_t a, row_t b, int d) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += elem(a, c) * elem(b, c);
    return acc;
}

/* ------------------------------------------------------- dropout hash */
/*
 * Counter-based dropout mask.  The pages only say that dropout is fused into
 * the kernel; the generator is this library's own definition:
 *   mix(x): x ^= x>>16; x *= C1; x ^= x>>15; x *= C2; x ^= x>>16   (mod 2^32)
 *   C1 = floor(frac(sqrt 2) * 2^32), C2 = floor(frac(sqrt 3) * 2^32),
 *   G  = floor(2^32 / golden ratio)
 *   row key  k_i = mix(mix(mix(mix(mix(lo(seed)^G) ^ hi(seed)) ^ b) ^ h) ^ i)
 *   pair     hash32(seed,b,h,i,u) = mix(k_i ^ (u*G)), u = j >> 1: one mix
 *            decides the two adjacent keys 2u and 2u+1 of row i
 *   element  h16(i,j) = low 16 bits of hash32(.., i, j >> 1) for even j,
 *            high 16 bits for odd j
 *   keep iff h16 >= T, T = ceil(p * 2^16) (0 <= T <= 2^16), so the keep
 *   probability (2^16 - T) / 2^16 is within 2^-16 of 1 - p.
 * The constants are derived here from their definitions, not typed in.
 */
static uint32_t C1, C2, G;
static int consts_ready = 0;

static void init_consts(void) {
    if (consts_ready) return;
    const double two32 = 4294967296.0;
    /* sqrt is correctly rounded in IEEE double; the products below are far
     * from an integer boundary, so floor() is exact. */
    C1 = (uint32_t)(uint64_t)floor((sqrt(2.0) - 1.0) * two32);
    C2 = (uint32_t)(uint64_t)floor((sqrt(3.0) - 1.0) * two32);
    G = (uint32_t)(uint64_t)floor(two32 / ((1.0 + sqrt(5.0)) / 2.0));
    consts_ready = 1;
}

static uint32_t mix32(uint32_t x) {
    x ^= x >> 16;
    x *= C1;
    x ^= x >> 15;
    x *= C2;
    x ^= x >> 16;
    return x;
}

uint32_t orc_hash_constant(int which) {
    init_consts();
    return which == 0 ? C1 : which == 1 ? C2 : G;
}

uint32_t orc_hash32(uint64_t seed, uint32_t b, uint32_t h, uint32_t i, uint32_t j) {
    init_consts();
    uint32_t key = mix32((uint32_t)seed ^ G);
    key = mix32(key ^ (uint32_t)(seed >> 32));
    key = mix32(key ^ b);
    key = mix32(key ^ h);
    key = mix32(key ^ i);
    return mix32(key ^ (j * G));
}

/* T = ceil(p * 2^16), compared with 16-bit hash halves; p in [0, 1). */
uint32_t orc_keep_threshold(double p) {
    double t = ceil(p * 65536.0);
    if (t <= 0.0) return 0u;
    if (t >= 65536.0) return 65536u;
    return (uint32_t)t;
}

static int keep_elem(const problem_t *pb, int bh, int i, int j) {
    if (pb->p_drop <= 0.0) return 1;
    uint32_t b = (uint32_t)(bh / pb->H), h = (uint32_t)(bh % pb->H);
    uint32_t w = orc_hash32(pb->seed, b, h, (uint32_t)i, (uint32_t)j >> 1);
    uint32_t h16 = (j & 1) ? (w >> 16) : (w & 0xffffu);
    return h16 >= orc_keep_threshold(pb->p_drop);
}

/* -------------------------------------------------------- one query row */

/* Is key j hidden from query i by the block mask? */
static int block_masked(const problem_t *pb, int bh, int i, int j) {
    if (!pb->bmask) return 0;
    const int nt = (pb->N + pb->bmask_tile - 1) / pb->bmask_tile;
    const int hm = pb->bmask_heads == 1 ? 0 : bh % pb->H;
    return pb->bmask[((size_t)hm * nt + (size_t)(i / pb->bmask_tile)) * nt + (size_t)(j / pb->bmask_tile)] == 0;
}

/* Number of real (non-padding) rows of the batch entry of head bh. */
static int seq_len(const problem_t *pb, int bh) {
    if (!pb->seqlens) return pb->N;
    const int L = pb->seqlens[bh / pb->H];
    return L < pb->N ? L : pb->N;
}

/* Scores s_ij for row i of head bh, then the row statistics m_i and l_i.
 * A row that sees no key (every key hidden by the block mask) has
 * m = -inf and l = 0; its probabilities are taken as 0. */
static void row_scores(const problem_t *pb, int bh, int i, double *s, double *m_out, double *l_out) {
    row_t qi = row_ptr(pb, pb->q, bh, i);
    const int L = seq_len(pb, bh);
    double m = -INFINITY;
    for (int j = 0; j < pb->N; ++j) {
        /* a padding query sees no key; a padding key is seen by no query */
        if (i >= L || j >= L || (pb->causal && j > i) || block_masked(pb, bh, i, j)) {
            s[j] = -INFINITY;
        } else {
            s[j] = pb->scale * dot_rows(qi, row_ptr(pb, pb->k, bh, j), pb->d);
        }
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    if (m != -INFINITY)
        for (int j = 0; j < pb->N; ++j) l += exp(s[j] - m); /* exp(-inf) = 0 */
    *m_out = m;
    *l_out = l;
}

/* P_ij for one score, from the row statistics (0 for a row with no key). */
static double prob(double s, double m, double l) { return l > 0.0 ? exp(s - m) / l : 0.0; }

/* O_i (d values) and lse_i for one query row. */
static void row_forward(const problem_t *pb, int bh, int i, double *s, double *o, double *lse) {
    double m, l;
    row_scores(pb, bh, i, s, &m, &l);
    const double inv_keep = 1.0 / (1.0 - pb->p_drop);
    for (int c = 0; c < pb->d; ++c) o[c] = 0.0;
    for (int j = 0; j < pb->N; ++j) {
        if (s[j] == -INFINITY) continue;
        double pd = prob(s[j], m, l) * (keep_elem(pb, bh, i, j) ? inv_keep : 0.0);
        if (pd == 0.0) continue;
        row_t vj = row_ptr(pb, pb->v, bh, j);
        for (int c = 0; c < pb->d; ++c) o[c] += pd * elem(vj, c);
    }
    *lse = l > 0.0 ? m + log(l) : -INFINITY;
}

/*
 * Backward quantities owned by query row i: D_i and dQ_i.  Also returns
 * <dO_i, O_i> so the caller can check the identity D_i = <dO_i, O_i>.
 */
static void row_backward_q(const problem_t *pb, int bh, int i, double *s, double *dq, double *D_out,
                           double *dot_do_o) {
    double m, l;
    row_scores(pb, bh, i, s, &m, &l);
    row_t doi = row_ptr(pb, pb->dout, bh, i);
    const double inv_keep = 1.0 / (1.0 - pb->p_drop);
    /* first pass: D_i = sum_j P_ij dP_ij and <dO_i, O_i> */
    double D = 0.0, doo = 0.0;
    for (int j = 0; j < pb->N; ++j) {
        if (s[j] == -INFINITY) continue;
        double p = prob(s[j], m, l);
        double z = keep_elem(pb, bh, i, j) ? inv_keep : 0.0;
        double dpd = dot_rows(doi, row_ptr(pb, pb->v, bh, j), pb->d); /* dO_i . v_j */
        D += p * (dpd * z);
        doo += (p * z) * dpd;
    }
    /* second pass: dS_ij and dQ_i */
    for (int c = 0; c < pb->d; ++c) dq[c] = 0.0;
    for (int j = 0; j < pb->N; ++j) {
        if (s[j] == -INFINITY) continue;
        double p = prob(s[j], m, l);
        double z = keep_elem(pb, bh, i, j) ? inv_keep : 0.0;
        double dp = dot_rows(doi, row_ptr(pb, pb->v, bh, j), pb->d) * z;
        double ds = p * (dp - D);
        row_t kj = row_ptr(pb, pb->k, bh, j);
        for (int c = 0; c < pb->d; ++c) dq[c] += ds * elem(kj, c);
    }
    for (int c = 0; c < pb->d; ++c) dq[c] *= pb->scale;
    *D_out = D;
    *dot_do_o = doo;
}

/* ------------------------------------------------------------- exports */

static problem_t make_problem(const void *q, const void *k, const void *v, const void *dout, int f64,
                             int B, int H, int N, int d, double scale, int causal, double p_drop,
                             uint64_t seed) {
    problem_t pb;
    pb.f64 = f64;
    pb.q = q;
    pb.k = k;
    pb.v = v;
    pb.dout = dout;
    pb.B = B;
    pb.H = H;
    pb.N = N;
    pb.d = d;
    pb.scale = scale;
    pb.causal = causal;
    pb.p_drop = p_drop;
    pb.seed = seed;
    pb.bmask = NULL;
    pb.bmask_heads = 1;
    pb.bmask_tile = 128;
    pb.seqlens = NULL;
    return pb;
}

/* Block mask used by the next orc_forward / orc_backward_q / orc_backward_kv
 * call of this thread (NULL: none).  mask is [heads][nt][nt] bytes with
 * nt = ceil(N / tile); heads is 1 (shared) or H. */
static _Thread_local const uint8_t *tl_bmask = NULL;
static _Thread_local int tl_bmask_heads = 1, tl_bmask_tile = 128;

void orc_set_block_mask(const uint8_t *mask, int heads, int tile) {
    tl_bmask = mask;
    tl_bmask_heads = heads;
    tl_bmask_tile = tile > 0 ? tile : 128;
}

/* Per-batch lengths used by the next calls of this thread (NULL: every
 * batch entry has all N rows).  lens is [B]. */
static _Thread_local const int32_t *tl_seqlens = NULL;

void orc_set_seqlens(const int32_t *lens) { tl_seqlens = lens; }

static void apply_block_mask(problem_t *pb) {
    pb->bmask = tl_bmask;
    pb->bmask_heads = tl_bmask_heads;
    pb->bmask_tile = tl_bmask_tile;
    pb->seqlens = tl_seqlens;
}

static int check_args(int B, int H, int N, int d, double p_drop) {
    if (B < 1 || H < 1 || N < 1 || d < 1) return -1;
    if (!(p_drop >= 0.0 && p_drop < 1.0)) return -1;
    return 0;
}

int orc_num_threads(void) { return omp_get_max_threads(); }

/*
 * Forward for the listed heads (bh = b*H + h) and query rows.  heads == NULL
 * means every head, rows == NULL every row.  Output o is
 * [nheads][nrows][d] and lse is [nheads][nrows] (natural log).
 */
int orc_forward(const void *q, const void *k, const void *v, int f64, int B, int H, int N, int d,
                double scale, int causal, double p_drop, uint64_t seed, const int32_t *heads, int nheads,
                const int32_t *rows, int nrows, double *o, double *lse) {
    if (check_args(B, H, N, d, p_drop)) return -1;
    init_consts();
    problem_t pb = make_problem(q, k, v, NULL, f64, B, H, N, d, scale, causal, p_drop, seed);
    apply_block_mask(&pb);
    int nh = heads ? nheads : B * H;
    int nr = rows ? nrows : N;
    int64_t total = (int64_t)nh * nr;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        if (!s) {
#pragma omp atomic write
            err = -2;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t u = 0; u < total; ++u) {
            if (!s) continue;
            int hi = (int)(u / nr), ri = (int)(u % nr);
            int bh = heads ? heads[hi] : hi;
            int i = rows ? rows[ri] : ri;
            row_forward(&pb, bh, i, s, o + (size_t)u * d, lse + u);
        }
        free(s);
    }
    return err;
}

/*
 * Query-side backward: dQ_i [nheads][nrows][d] and D_i [nheads][nrows] for
 * the listed heads/rows.  max_rel_dev receives the largest
 * |D_i - <dO_i,O_i>| / max(1, |D_i|) seen (an internal consistency check).
 */
int orc_backward_q(const void *q, const void *k, const void *v, const void *dout, int f64, int B,
                   int H, int N, int d, double scale, int causal, double p_drop, uint64_t seed,
                   const int32_t *heads, int nheads, const int32_t *rows, int nrows, double *dq, double *D,
                   double *max_rel_dev) {
    if (check_args(B, H, N, d, p_drop)) return -1;
    init_consts();
    problem_t pb = make_problem(q, k, v, dout, f64, B, H, N, d, scale, causal, p_drop, seed);
    apply_block_mask(&pb);
    int nh = heads ? nheads : B * H;
    int nr = rows ? nrows : N;
    int64_t total = (int64_t)nh * nr;
    double worst = 0.0;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double local_worst = 0.0;
        if (!s) {
#pragma omp atomic write
            err = -2;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t u = 0; u < total; ++u) {
            if (!s) continue;
            int hi = (int)(u / nr), ri = (int)(u % nr);
            int bh = heads ? heads[hi] : hi;
            int i = rows ? rows[ri] : ri;
            double doo;
            row_backward_q(&pb, bh, i, s, dq + (size_t)u * d, D + u, &doo);
            double dev = fabs(D[u] - doo) / fmax(1.0, fabs(D[u]));
            if (dev > local_worst) local_worst = dev;
        }
#pragma omp critical
        {
            if (local_worst > worst) worst = local_worst;
        }
        free(s);
    }
    if (max_rel_dev) *max_rel_dev = worst;
    return err;
}

/*
 * Key-side backward: dK_j and dV_j [nheads][nkeys][d] for the listed heads
 * and key rows.  Each needs m_i, l_i and D_i of every query row i that sees
 * key j, so a full statistics pass over those query rows runs first (O(N^2 d)
 * per head); with a causal mask only rows i >= min(keys) are visited.
 */
int orc_backward_kv(const void *q, const void *k, const void *v, const void *dout, int f64, int B,
                    int H, int N, int d, double scale, int causal, double p_drop, uint64_t seed,
                    const int32_t *heads, int nheads, const int32_t *keys, int nkeys, double *dk, double *dv) {
    if (check_args(B, H, N, d, p_drop)) return -1;
    init_consts();
    problem_t pb = make_problem(q, k, v, dout, f64, B, H, N, d, scale, causal, p_drop, seed);
    apply_block_mask(&pb);
    int nh = heads ? nheads : B * H;
    int nk = keys ? nkeys : N;
    int first_row = 0;
    if (causal) {
        first_row = N;
        for (int t = 0; t < nk; ++t) {
            int j = keys ? keys[t] : t;
            if (j < first_row) first_row = j;
        }
    }
    int nstat = N - first_row;
    double *m = (double *)malloc(sizeof(double) * (size_t)nh * (size_t)(nstat > 0 ? nstat : 1));
    double *l = (double *)malloc(sizeof(double) * (size_t)nh * (size_t)(nstat > 0 ? nstat : 1));
    double *D = (double *)malloc(sizeof(double) * (size_t)nh * (size_t)(nstat > 0 ? nstat : 1));
    if (!m || !l || !D) {
        free(m);
        free(l);
        free(D);
        return -2;
    }
    int err = 0;
    const double inv_keep = 1.0 / (1.0 - p_drop);
    /* statistics pass: m_i, l_i, D_i for rows first_row..N-1 */
    int64_t total = (int64_t)nh * nstat;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        if (!s) {
#pragma omp atomic write
            err = -2;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t u = 0; u < total; ++u) {
            if (!s) continue;
            int hi = (int)(u / nstat);
            int i = first_row + (int)(u % nstat);
            int bh = heads ? heads[hi] : hi;
            double mi, li;
            row_scores(&pb, bh, i, s, &mi, &li);
            row_t doi = row_ptr(&pb, pb.dout, bh, i);
            double Di = 0.0;
            for (int j = 0; j < N; ++j) {
                if (s[j] == -INFINITY) continue;
                double z = keep_elem(&pb, bh, i, j) ? inv_keep : 0.0;
                double dp = dot_rows(doi, row_ptr(&pb, pb.v, bh, j), d) * z;
                Di += prob(s[j], mi, li) * dp;
            }
            m[u] = mi;
            l[u] = li;
            D[u] = Di;
        }
        free(s);
    }
    if (err) {
        free(m);
        free(l);
        free(D);
        return err;
    }
    /* key pass: dV_j = sum_i Pd_ij dO_i ; dK_j = scale * sum_i dS_ij q_i */
    int64_t ktotal = (int64_t)nh * nk;
#pragma omp parallel for schedule(dynamic, 2)
    for (int64_t u = 0; u < ktotal; ++u) {
        int hi = (int)(u / nk), ki = (int)(u % nk);
        int bh = heads ? heads[hi] : hi;
        int j = keys ? keys[ki] : ki;
        double *dkj = dk + (size_t)u * d;
        double *dvj = dv + (size_t)u * d;
        for (int c = 0; c < d; ++c) {
            dkj[c] = 0.0;
            dvj[c] = 0.0;
        }
        const int L = seq_len(&pb, bh);
        if (j >= L) continue; /* a padding key: dK_j = dV_j = 0 */
        row_t kj = row_ptr(&pb, pb.k, bh, j);
        row_t vj = row_ptr(&pb, pb.v, bh, j);
        int i0 = causal ? j : 0;
        for (int i = i0; i < L; ++i) {
            if (block_masked(&pb, bh, i, j)) continue;
            size_t su = (size_t)hi * nstat + (size_t)(i - first_row);
            row_t qi = row_ptr(&pb, pb.q, bh, i);
            row_t doi = row_ptr(&pb, pb.dout, bh, i);
            double sij = scale * dot_rows(qi, kj, d);
            double p = prob(sij, m[su], l[su]);
            double z = keep_elem(&pb, bh, i, j) ? inv_keep : 0.0;
            double dp = dot_rows(doi, vj, d) * z;
            double ds = p * (dp - D[su]);
            double pd = p * z;
            for (int c = 0; c < d; ++c) {
                dvj[c] += pd * elem(doi, c);
                dkj[c] += ds * elem(qi, c);
            }
        }
        for (int c = 0; c < d; ++c) dkj[c] *= scale;
    }
    free(m);
    free(l);
    free(D);
    return 0;
}

/* Dropout keep bits (1 = kept) for the listed heads/rows over all N keys:
 * out is [nheads][nrows][N] bytes. */
int orc_dropout_mask(int B, int H, int N, double p_drop, uint64_t seed, const int32_t *heads, int nheads,
                     const int32_t *rows, int nrows, uint8_t *out) {
    if (check_args(B, H, N, 1, p_drop)) return -1;
    init_consts();
    problem_t pb = make_problem(NULL, NULL, NULL, NULL, 0, B, H, N, 1, 1.0, 0, p_drop, seed);
    int nh = heads ? nheads : B * H;
    int nr = rows ? nrows : N;
    int64_t total = (int64_t)nh * nr;
#pragma omp parallel for schedule(static)
    for (int64_t u = 0; u < total; ++u) {
        int hi = (int)(u / nr), ri = (int)(u % nr);
        int bh = heads ? heads[hi] : hi;
        int i = rows ? rows[ri] : ri;
        for (int j = 0; j < N; ++j) out[(size_t)u * N + j] = (uint8_t)keep_elem(&pb, bh, i, j);
    }
    return 0;
}
