/*
 * oracle.c -- plain fp64 CPU oracle for block-causal linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent checker of the CUDA
 * library; only the tests, the smoke check and the benchmark's CPU-baseline leg
 * may load it.  It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes (notation of the pages):
 *   Sources, cited by page title and section:
 *   [aihaber]    "Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı"
 *                (aihaber.org), sections "Verimli doğrusal DiT" and
 *                "Sabit Bellekli KV önbelleğe alma mekanizması".
 *   [sd114]      sd114.wiki SANA-Video summary, section "两大核心技术突破",
 *                item 1 (线性 DiT, incl. RoPE) and item 2 (块线性注意力 + 恒定内存 KV 缓存).
 *   [chatpaper]  "SANA-Video: Efficient Video Generation with Block Linear
 *                Diffusion Transformer", abstract (chatpaper.ai), design (2).
 *
 *   Linear attention replaces softmax by a kernel feature map phi and a global
 *   aggregation, so no N x N matrix is formed [sd114 item 1; aihaber
 *   "Verimli doğrusal DiT"].  phi = ReLU.
 *   The video is split into blocks along time; later blocks see earlier ones,
 *   never the reverse; tokens inside a block see each other [aihaber
 *   "Sabit Bellekli ..." paragraphs 2 and 5].
 *   Per head and block n:  KV_n = sum_{t in n} psi(k_t)^T v_t  (d x d),
 *                          z_n  = sum_{t in n} phi(k_t)         (d),
 *   the cached state is S_{n-1} = KV_1 + ... + KV_{n-1}, Z_{n-1} likewise
 *   ("KV_{1-2} = KV_1 + KV_2", constant size [aihaber para 4; sd114 item 2]),
 *   and each token of block n gets
 *        out = psi(q) (S_{n-1} + KV_n) / ( phi(q) . (Z_{n-1} + z_n) + eps ).
 *   psi = phi without RoPE; with RoPE psi = R(position) o phi in the numerator
 *   only, the denominator stays unrotated ([sd114 item 1] names RoPE; its
 *   placement, pairing and frequencies are a stated reading, see below).
 *
 *   RoPE reading: the d features are cut into three sections of dt, dh, dw
 *   dims for the latent frame, row and column of the token.  Inside a section
 *   of D dims, features (2i, 2i+1) form a pair rotated by the angle
 *   pos * base^(-2i/D):  x'_{2i} = x_{2i} cos - x_{2i+1} sin,
 *                        x'_{2i+1} = x_{2i} sin + x_{2i+1} cos.
 *   Token j of a call (counted from tok_base) sits at frame
 *   t_offset + j / (Hg*Wg), row (j % (Hg*Wg)) / Wg, column j % Wg.
 *
 * Two independent forms are provided:
 *   orc_brute      -- the definition: out_i = sum_{j: blk(j) <= blk(i)}
 *                     (psi(q_i).psi(k_j)) v_j / (sum phi(q_i).phi(k_j) + eps).
 *                     O(N^2 d) per head.
 *   orc_block_kv / orc_apply / orc_block_forward / orc_full_forward
 *                  -- the recurrence of the method, step by step.
 *
 * Inputs are read in their stored type (fp64, fp32, or bf16 bit patterns) and
 * widened exactly to fp64; every sum and product is fp64.  Layout of q, k, v,
 * out: [B][N][H][d], d fastest.  State S: [B][H][d][d] (row = key feature,
 * column = value feature), Z: [B][H][d].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

typedef struct {
    int enabled;   /* 0: psi = phi */
    int Hg, Wg;    /* latent grid rows and columns; one frame = Hg*Wg tokens */
    int t_offset;  /* latent frame of token 0 of the call */
    int dt, dh, dw;/* dims per axis section, dt + dh + dw == d, each even */
    double base;   /* frequency base */
} orc_rope;

/* Widen one stored element to fp64.  bf16 is the top half of an fp32. */
static double elem(const void *p, int dtype, size_t i)
{
    if (dtype == ORC_F64) return ((const double *)p)[i];
    if (dtype == ORC_F32) return (double)((const float *)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static size_t idx4(int b, long t, int h, int e, long N, int H, int d)
{
    return (((size_t)b * (size_t)N + (size_t)t) * (size_t)H + (size_t)h) * (size_t)d + (size_t)e;
}

/* phi = ReLU, elementwise, on the d features of token t, head h. */
static void phi_row(const void *x, int dtype, int b, long t, int h, long N, int H, int d, double *f)
{
    for (int e = 0; e < d; ++e) {
        double a = elem(x, dtype, idx4(b, t, h, e, N, H, d));
        f[e] = a > 0.0 ? a : 0.0;
    }
}

/* Rotate one section [lo, lo+D) of f by position pos (interleaved pairs). */
static void rotate_section(double *f, int lo, int D, long pos, double base)
{
    for (int i = 0; i < D / 2; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)D);
        double ang = (double)pos * theta;
        double c = cos(ang), s = sin(ang);
        double x0 = f[lo + 2 * i], x1 = f[lo + 2 * i + 1];
        f[lo + 2 * i] = x0 * c - x1 * s;
        f[lo + 2 * i + 1] = x0 * s + x1 * c;
    }
}

/* psi(f) for token number j of the call: f -> R(pos(j)) f, in place. */
static void rope_apply(double *f, const orc_rope *r, long j)
{
    if (!r || !r->enabled) return;
    long per_frame = (long)r->Hg * (long)r->Wg;
    long tpos = (long)r->t_offset + j / per_frame;
    long rem = j % per_frame;
    long hpos = rem / r->Wg;
    long wpos = rem % r->Wg;
    rotate_section(f, 0, r->dt, tpos, r->base);
    rotate_section(f, r->dt, r->dh, hpos, r->base);
    rotate_section(f, r->dt + r->dh, r->dw, wpos, r->base);
}

static int rope_ok(const orc_rope *r, int d)
{
    if (!r || !r->enabled) return 1;
    if (r->Hg <= 0 || r->Wg <= 0) return 0;
    if (r->dt < 0 || r->dh < 0 || r->dw < 0) return 0;
    if ((r->dt | r->dh | r->dw) & 1) return 0;
    return r->dt + r->dh + r->dw == d;
}

static int threads_wanted = 0;

void orc_set_threads(int n) { threads_wanted = n; }

int orc_get_threads(void)
{
#ifdef _OPENMP
    return threads_wanted > 0 ? threads_wanted : omp_get_max_threads();
#else
    return 1;
#endif
}

#ifdef _OPENMP
#define ORC_THREADS num_threads(orc_get_threads())
#endif

/*
 * Definition form.  Token i of block blk(i) = i / L (L = tokens_per_block, 0 means
 * one block of all N tokens) attends to every token j with blk(j) <= blk(i).
 */
int orc_brute(const void *q, const void *k, const void *v, int dtype, double *out,
              int B, long N, int H, int d, long tokens_per_block,
              const orc_rope *rope, long tok_base, double eps)
{
    if (B < 0 || N < 0 || H < 0 || d <= 0 || d > 256 || tokens_per_block < 0) return 1;
    if (!rope_ok(rope, d)) return 1;
    long L = tokens_per_block > 0 ? tokens_per_block : (N > 0 ? N : 1);
    long total = (long)B * H * N;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 16) ORC_THREADS
#endif
    for (long w = 0; w < total; ++w) {
        int b = (int)(w / ((long)H * N));
        long i = (w / H) % N;
        int h = (int)(w % H);
        double fq[256], pq[256], fk[256], pk[256], num[256];
        phi_row(q, dtype, b, i, h, N, H, d, fq);
        memcpy(pq, fq, sizeof(double) * d);
        rope_apply(pq, rope, tok_base + i);
        for (int e = 0; e < d; ++e) num[e] = 0.0;
        double den = 0.0;
        long last = (i / L + 1) * L;           /* end of i's block (exclusive) */
        if (last > N) last = N;
        for (long j = 0; j < last; ++j) {
            phi_row(k, dtype, b, j, h, N, H, d, fk);
            memcpy(pk, fk, sizeof(double) * d);
            rope_apply(pk, rope, tok_base + j);
            double a_num = 0.0, a_den = 0.0;
            for (int e = 0; e < d; ++e) {
                a_num += pq[e] * pk[e];
                a_den += fq[e] * fk[e];
            }
            for (int e = 0; e < d; ++e) num[e] += a_num * elem(v, dtype, idx4(b, j, h, e, N, H, d));
            den += a_den;
        }
        for (int e = 0; e < d; ++e) out[idx4(b, i, h, e, N, H, d)] = num[e] / (den + eps);
    }
    return 0;
}

/*
 * KV_n and z_n of the tokens [t0, t1) of a call ("KV product then accumulate",
 * [aihaber "Sabit Bellekli ..." para 3]):
 *   KV[b][h][a][c] = sum_t psi(k_t)[a] v_t[c],   z[b][h][a] = sum_t phi(k_t)[a].
 * Positions for RoPE are tok_base + t.
 */
int orc_block_kv(const void *k, const void *v, int dtype, int B, long N, int H, int d,
                 long t0, long t1, const orc_rope *rope, long tok_base,
                 double *KV, double *z)
{
    if (B < 0 || N < 0 || H < 0 || d <= 0 || d > 256) return 1;
    if (t0 < 0 || t1 > N || t0 > t1) return 1;
    if (!rope_ok(rope, d)) return 1;
    long pairs = (long)B * H;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) ORC_THREADS
#endif
    for (long w = 0; w < pairs; ++w) {
        int b = (int)(w / H), h = (int)(w % H);
        double *kv = KV + (size_t)w * d * d;
        double *zz = z + (size_t)w * d;
        double fk[256], pk[256];
        for (int a = 0; a < d * d; ++a) kv[a] = 0.0;
        for (int a = 0; a < d; ++a) zz[a] = 0.0;
        for (long t = t0; t < t1; ++t) {
            phi_row(k, dtype, b, t, h, N, H, d, fk);
            memcpy(pk, fk, sizeof(double) * d);
            rope_apply(pk, rope, tok_base + t);
            for (int a = 0; a < d; ++a) {
                zz[a] += fk[a];
                for (int c = 0; c < d; ++c)
                    kv[(size_t)a * d + c] += pk[a] * elem(v, dtype, idx4(b, t, h, c, N, H, d));
            }
        }
    }
    return 0;
}

/*
 * out_t = psi(q_t) S_eff / (phi(q_t) . Z_eff + eps) for the listed tokens
 * ("each block needs only KVsum plus its own KV", [aihaber "Sabit Bellekli ..."
 * last para]).  S_eff [B][H][d][d], Z_eff [B][H][d].  out is [B][ntok][H][d]
 * in the order of toks.
 */
int orc_apply(const void *q, int dtype, int B, long N, int H, int d,
              const double *S_eff, const double *Z_eff, const long *toks, long ntok,
              const orc_rope *rope, long tok_base, double eps, double *out)
{
    if (B < 0 || N < 0 || H < 0 || d <= 0 || d > 256 || ntok < 0) return 1;
    if (!rope_ok(rope, d)) return 1;
    for (long m = 0; m < ntok; ++m)
        if (toks[m] < 0 || toks[m] >= N) return 1;
    long total = (long)B * ntok * H;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) ORC_THREADS
#endif
    for (long w = 0; w < total; ++w) {
        int b = (int)(w / ((long)ntok * H));
        long m = (w / H) % ntok;
        int h = (int)(w % H);
        long t = toks[m];
        const double *S = S_eff + ((size_t)b * H + h) * d * d;
        const double *Z = Z_eff + ((size_t)b * H + h) * d;
        double fq[256], pq[256];
        phi_row(q, dtype, b, t, h, N, H, d, fq);
        memcpy(pq, fq, sizeof(double) * d);
        rope_apply(pq, rope, tok_base + t);
        double den = 0.0;
        for (int a = 0; a < d; ++a) den += fq[a] * Z[a];
        for (int c = 0; c < d; ++c) {
            double num = 0.0;
            for (int a = 0; a < d; ++a) num += pq[a] * S[(size_t)a * d + c];
            out[idx4(b, m, h, c, ntok, H, d)] = num / (den + eps);
        }
    }
    return 0;
}

/*
 * One block of the streaming method: KV_n, z_n over the call's N tokens, then
 * S_eff = S + KV_n, Z_eff = Z + z_n, out for every token, and, if commit,
 * S <- S_eff, Z <- Z_eff ("cache KV_1; when KV_2 is done add it to get KV_{1-2}",
 * [aihaber "Sabit Bellekli ..." para 4]).  S, Z are this oracle's own fp64 state.
 */
int orc_block_forward(const void *q, const void *k, const void *v, int dtype, double *out,
                      int B, long N, int H, int d, double *S, double *Z, int commit,
                      const orc_rope *rope, long tok_base, double eps)
{
    if (B < 0 || N < 0 || H < 0 || d <= 0 || d > 256) return 1;
    size_t nS = (size_t)B * H * d * d, nZ = (size_t)B * H * d;
    double *KV = malloc(sizeof(double) * (nS + 1));
    double *z = malloc(sizeof(double) * (nZ + 1));
    double *Se = malloc(sizeof(double) * (nS + 1));
    double *Ze = malloc(sizeof(double) * (nZ + 1));
    long *toks = malloc(sizeof(long) * (size_t)(N + 1));
    int rc = 1;
    if (!KV || !z || !Se || !Ze || !toks) goto done;
    rc = orc_block_kv(k, v, dtype, B, N, H, d, 0, N, rope, tok_base, KV, z);
    if (rc) goto done;
    for (size_t a = 0; a < nS; ++a) Se[a] = S[a] + KV[a];
    for (size_t a = 0; a < nZ; ++a) Ze[a] = Z[a] + z[a];
    for (long t = 0; t < N; ++t) toks[t] = t;
    rc = orc_apply(q, dtype, B, N, H, d, Se, Ze, toks, N, rope, tok_base, eps, out);
    if (rc) goto done;
    if (commit) {
        memcpy(S, Se, sizeof(double) * nS);
        memcpy(Z, Ze, sizeof(double) * nZ);
    }
done:
    free(KV); free(z); free(Se); free(Ze); free(toks);
    return rc;
}

/*
 * A whole sequence from a zero state: blocks of L = tokens_per_block tokens
 * (0: one block of N; the last block may be shorter), each run as one
 * orc_block_forward with commit, positions continuing across blocks.
 * Works on [B][N][H][d] by copying each block's slice out (plain, not fast).
 */
int orc_full_forward(const void *q, const void *k, const void *v, int dtype, double *out,
                     int B, long N, int H, int d, long tokens_per_block,
                     const orc_rope *rope, double eps)
{
    if (B < 0 || N < 0 || H < 0 || d <= 0 || d > 256 || tokens_per_block < 0) return 1;
    long L = tokens_per_block > 0 ? tokens_per_block : (N > 0 ? N : 1);
    size_t es = dtype == ORC_F64 ? 8 : dtype == ORC_F32 ? 4 : 2;
    size_t nS = (size_t)B * H * d * d, nZ = (size_t)B * H * d;
    double *S = calloc(nS + 1, sizeof(double));
    double *Z = calloc(nZ + 1, sizeof(double));
    size_t row = (size_t)H * d;             /* elements per token */
    size_t maxblk = (size_t)B * (size_t)L * row;
    unsigned char *qb = malloc(es * maxblk + 1), *kb = malloc(es * maxblk + 1), *vb = malloc(es * maxblk + 1);
    double *ob = malloc(sizeof(double) * maxblk + 1);
    int rc = 1;
    if (!S || !Z || !qb || !kb || !vb || !ob) goto done;
    rc = 0;
    for (long t0 = 0; t0 < N && rc == 0; t0 += L) {
        long n = (t0 + L <= N) ? L : N - t0;
        for (int b = 0; b < B; ++b) {
            size_t src = ((size_t)b * N + t0) * row * es, dst = (size_t)b * n * row * es;
            memcpy(qb + dst, (const unsigned char *)q + src, (size_t)n * row * es);
            memcpy(kb + dst, (const unsigned char *)k + src, (size_t)n * row * es);
            memcpy(vb + dst, (const unsigned char *)v + src, (size_t)n * row * es);
        }
        rc = orc_block_forward(qb, kb, vb, dtype, ob, B, n, H, d, S, Z, 1, rope, t0, eps);
        for (int b = 0; b < B && rc == 0; ++b)
            memcpy(out + ((size_t)b * N + t0) * row, ob + (size_t)b * n * row, sizeof(double) * (size_t)n * row);
    }
done:
    free(S); free(Z); free(qb); free(kb); free(vb); free(ob);
    return rc;
}

/* psi^T: the transpose of rope_apply (rotation by the negative angle). */
static void rope_apply_t(double *f, const orc_rope *r, long j)
{
    if (!r || !r->enabled) return;
    long per_frame = (long)r->Hg * (long)r->Wg;
    long tpos = (long)r->t_offset + j / per_frame;
    long rem = j % per_frame;
    rotate_section(f, 0, r->dt, -tpos, r->base);
    rotate_section(f, r->dt, r->dh, -(rem / r->Wg), r->base);
    rotate_section(f, r->dt + r->dh, r->dw, -(rem % r->Wg), r->base);
}

/*
 * Gradient of orc_full_forward (zero initial state, blocks of
 * tokens_per_block tokens): with dout [B][N][H][d] given, dq, dk, dv
 * [B][N][H][d] are the gradients of sum(out * dout) with respect to q, k, v.
 * The chain rule through the recurrence of the method, per (b, h):
 *   forward:  S_n = sum_{m<=n} KV_m, Z_n = sum_{m<=n} z_m (inclusive)
 *   block n, token t:  num_t = psi(q_t) S_n,  den_t = phi(q_t) . Z_n + eps,
 *     g_t = dout_t / den_t,  c_t = -(dout_t . num_t) / den_t^2,
 *     d psi(q_t) = S_n g_t,  d phi(q_t) += c_t Z_n,
 *     dS_n += psi(q_t) g_t^T,  dZ_n += c_t phi(q_t)
 *   the state of block m enters every later block:
 *     G_m = sum_{n>=m} dS_n,  g_m = sum_{n>=m} dZ_n
 *   block m, token t:  d psi(k_t) = G_m v_t,  dv_t = G_m^T psi(k_t),
 *     d phi(k_t) += g_m
 *   then d phi = R^T d psi (+ the unrotated part) and the ReLU mask 1[x > 0].
 * The pages state only the forward recurrence ([aihaber "Sabit Bellekli ..."]);
 * the backward is its derivative, for block-autoregressive training.
 */
int orc_full_backward(const void *q, const void *k, const void *v, const void *dout, int dtype,
                      double *dq, double *dk, double *dv, int B, long N, int H, int d,
                      long tokens_per_block, const orc_rope *rope, double eps)
{
    if (B < 0 || N < 0 || H < 0 || d <= 0 || d > 256 || tokens_per_block < 0) return 1;
    if (!rope_ok(rope, d)) return 1;
    long L = tokens_per_block > 0 ? tokens_per_block : (N > 0 ? N : 1);
    long nb = N > 0 ? (N + L - 1) / L : 0;
    long total = (long)B * H;
    int bad = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) ORC_THREADS reduction(| : bad)
#endif
    for (long w = 0; w < total; ++w) {
        int b = (int)(w / H), h = (int)(w % H);
        size_t dd = (size_t)d * d;
        double *S = calloc((size_t)nb * dd + 1, sizeof(double));
        double *Z = calloc((size_t)nb * d + 1, sizeof(double));
        double *dS = calloc((size_t)nb * dd + 1, sizeof(double));
        double *dZ = calloc((size_t)nb * d + 1, sizeof(double));
        double *G = calloc(dd + 1, sizeof(double));
        double *gz = calloc((size_t)d + 1, sizeof(double));
        if (!S || !Z || !dS || !dZ || !G || !gz) {
            bad = 1;
            goto next;
        }
        double f[256], p[256], dp[256], df[256], num[256], g[256];
        /* forward prefix: S_n, Z_n after block n */
        for (long n = 0; n < nb; ++n) {
            double *Sn = S + (size_t)n * dd, *Zn = Z + (size_t)n * d;
            if (n > 0) {
                memcpy(Sn, Sn - dd, sizeof(double) * dd);
                memcpy(Zn, Zn - d, sizeof(double) * d);
            }
            long t1 = (n + 1) * L < N ? (n + 1) * L : N;
            for (long t = n * L; t < t1; ++t) {
                phi_row(k, dtype, b, t, h, N, H, d, f);
                memcpy(p, f, sizeof(double) * d);
                rope_apply(p, rope, t);
                for (int a = 0; a < d; ++a) {
                    Zn[a] += f[a];
                    for (int c = 0; c < d; ++c) Sn[(size_t)a * d + c] += p[a] * elem(v, dtype, idx4(b, t, h, c, N, H, d));
                }
            }
        }
        /* query side: dq, dS_n, dZ_n */
        for (long n = 0; n < nb; ++n) {
            const double *Sn = S + (size_t)n * dd, *Zn = Z + (size_t)n * d;
            double *dSn = dS + (size_t)n * dd, *dZn = dZ + (size_t)n * d;
            long t1 = (n + 1) * L < N ? (n + 1) * L : N;
            for (long t = n * L; t < t1; ++t) {
                phi_row(q, dtype, b, t, h, N, H, d, f);
                memcpy(p, f, sizeof(double) * d);
                rope_apply(p, rope, t);
                double den = eps, dn = 0.0;
                for (int a = 0; a < d; ++a) den += f[a] * Zn[a];
                for (int c = 0; c < d; ++c) {
                    num[c] = 0.0;
                    for (int a = 0; a < d; ++a) num[c] += p[a] * Sn[(size_t)a * d + c];
                    double o = elem(dout, dtype, idx4(b, t, h, c, N, H, d));
                    g[c] = o / den;
                    dn += o * num[c];
                }
                double cc = -dn / (den * den);
                for (int a = 0; a < d; ++a) {
                    dp[a] = 0.0;
                    for (int c = 0; c < d; ++c) dp[a] += Sn[(size_t)a * d + c] * g[c];
                }
                memcpy(df, dp, sizeof(double) * d);
                rope_apply_t(df, rope, t);
                for (int a = 0; a < d; ++a) {
                    df[a] += cc * Zn[a];
                    double x = elem(q, dtype, idx4(b, t, h, a, N, H, d));
                    dq[idx4(b, t, h, a, N, H, d)] = x > 0.0 ? df[a] : 0.0;
                    dZn[a] += cc * f[a];
                    for (int c = 0; c < d; ++c) dSn[(size_t)a * d + c] += p[a] * g[c];
                }
            }
        }
        /* key side, last block first: G_m = sum_{n>=m} dS_n */
        for (long m = nb - 1; m >= 0; --m) {
            for (size_t a = 0; a < dd; ++a) G[a] += dS[(size_t)m * dd + a];
            for (int a = 0; a < d; ++a) gz[a] += dZ[(size_t)m * d + a];
            long t1 = (m + 1) * L < N ? (m + 1) * L : N;
            for (long t = m * L; t < t1; ++t) {
                phi_row(k, dtype, b, t, h, N, H, d, f);
                memcpy(p, f, sizeof(double) * d);
                rope_apply(p, rope, t);
                for (int a = 0; a < d; ++a) {
                    dp[a] = 0.0;
                    for (int c = 0; c < d; ++c) dp[a] += G[(size_t)a * d + c] * elem(v, dtype, idx4(b, t, h, c, N, H, d));
                }
                for (int c = 0; c < d; ++c) {
                    double s = 0.0;
                    for (int a = 0; a < d; ++a) s += G[(size_t)a * d + c] * p[a];
                    dv[idx4(b, t, h, c, N, H, d)] = s;
                }
                memcpy(df, dp, sizeof(double) * d);
                rope_apply_t(df, rope, t);
                for (int a = 0; a < d; ++a) {
                    df[a] += gz[a];
                    double x = elem(k, dtype, idx4(b, t, h, a, N, H, d));
                    dk[idx4(b, t, h, a, N, H, d)] = x > 0.0 ? df[a] : 0.0;
                }
            }
        }
    next:
        free(S); free(Z); free(dS); free(dZ); free(G); free(gz);
    }
    return bad;
}

/*
 * Depthwise 3D convolution of the Spatial-Temporal Mix-FFN ("Nvidia, MIT ve
 * diğerleri video yapay zeka devrimini başlattı", section "Verimli doğrusal
 * DiT": the MLP alternates a 1x3x3 spatial and a 3x1x1 temporal convolution to
 * add local information to each token).  x, y are [B][T][Hg][Wg][C] (tokens in
 * frame, row, column order, channels last), w is [C][kt][kh][kw], bias [C] or
 * NULL; odd kernel sizes, zero padding of (k-1)/2 on each side, within the
 * call's frames:
 *   y[b,t,h,w,c] = bias[c] + sum_{i,j,l} w[c][i][j][l] x[b, t+i-pt, h+j-ph, w+l-pw, c]
 * with out-of-range taps reading 0.
 */
int orc_dwconv3d(const void *x, int dtype, double *y, int B, int T, int Hg, int Wg, int C,
                 int kt, int kh, int kw, const double *w, const double *bias)
{
    if (B < 0 || T < 0 || Hg < 0 || Wg < 0 || C <= 0) return 1;
    if (kt < 1 || kh < 1 || kw < 1 || !(kt & 1) || !(kh & 1) || !(kw & 1)) return 1;
    int pt = kt / 2, ph = kh / 2, pw = kw / 2;
    long ntok = (long)B * T * Hg * Wg;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) ORC_THREADS
#endif
    for (long tok = 0; tok < ntok; ++tok) {
        long r = tok;
        int ww = (int)(r % Wg); r /= Wg;
        int hh = (int)(r % Hg); r /= Hg;
        int tt = (int)(r % T); r /= T;
        int b = (int)r;
        for (int c = 0; c < C; ++c) {
            double acc = bias ? bias[c] : 0.0;
            for (int i = 0; i < kt; ++i) {
                int t2 = tt + i - pt;
                if (t2 < 0 || t2 >= T) continue;
                for (int j = 0; j < kh; ++j) {
                    int h2 = hh + j - ph;
                    if (h2 < 0 || h2 >= Hg) continue;
                    for (int l = 0; l < kw; ++l) {
                        int w2 = ww + l - pw;
                        if (w2 < 0 || w2 >= Wg) continue;
                        size_t src = ((((size_t)b * T + t2) * Hg + h2) * Wg + w2) * C + c;
                        acc += w[(((size_t)c * kt + i) * kh + j) * kw + l] * elem(x, dtype, src);
                    }
                }
            }
            y[(size_t)tok * C + c] = acc;
        }
    }
    return 0;
}
