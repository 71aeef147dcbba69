/*
 * Window-attention oracle: a plain, slow, fp64 CPU statement of what the
 * fused window-attention forward computes.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline of the benchmark may load this library.  It shares no code,
 * header, table or helper with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it follows (pages are cited by title and section):
 *  - "FLASHSWIN: Unlocking Large Windows and Dense Tokens in Swin Vision
 *    Transformers with Memory Efficient Attention", section "어떻게 동작하나"
 *    (how it works): attention is exact softmax attention restricted to
 *    non-overlapping M x M windows; shifted windows are a cyclic move of the
 *    map followed by per-window recomputation; wrapped windows are masked by
 *    an additive mask; window-local learned 2D RoPE splits the head dim in
 *    half, the first half encoding the row y and the second half the column
 *    x, both halves sharing one frequency set theta_i = exp(omega_i).
 *  - same page, section "전제와 한계" (premises and limits), second
 *    paragraph: bf16 Q/K/V in, RoPE in fp32, softmax accumulated in fp32
 *    (the oracle does all of it in fp64 on the exact input values).
 *  - "Rank-Factorized Implicit Neural Bias: Scaling Super-Resolution
 *    Transformer with FlashAttention", section 2.1 (RIB): the position
 *    features are concatenated to the content features so that
 *    [Qc, Qp][Kc, Kp]^T = Qc Kc^T + Qp Kp^T.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - d/4 shared frequencies per head (the page's "d/2 parameters per head"
 *    cannot rotate d/2 dims with one angle per pair); pairs are adjacent
 *    (2k, 2k+1) inside each half; counter-clockwise rotation;
 *  - roll by -s (token (i, j) of the rolled map is original token
 *    (i + s, j + s) mod (H, W)), inverse roll on write-back;
 *  - wrap label L = 2*[row in last s rows] + [col in last s cols] of the
 *    rolled map, mask value -inf where labels differ;
 *  - maps whose sides are not multiples of M (FlashSwin-T's 56 x 56 map at
 *    M = 16 or 32) are padded at the bottom and right to the next multiples
 *    Hp x Wp, the padded map is rolled and cut into windows (Swin pads before
 *    its roll), and the pad positions hold no token: they are masked as keys
 *    (-inf) and never written; the labels above use Hp and Wp;
 *  - scale d^-1/2 applies to the content dot product only, the bias dot
 *    product u.w is added unscaled.
 *
 * Parity of every function here is pinned by the not-gpu tests (closed
 * forms, the displacement identity of the rotation, brute-force masked
 * global attention, Swin's slice-based region labels, planted mistakes).
 *
 * The gated residual (oracle_fwd_sparse) follows "HSMLA: Hierarchical
 * Softmax Multi-scale Linear Attention for Efficient Vision Transformers",
 * section 2 (방법론), "Hierarchical Block-Level Gating" and "Two-Path
 * Residual Kernel": every token keeps the global linear-attention output
 * O_lin; only the gated blocks (here: windows) also run the local softmax
 * attention, and add the residual O_local - O_lin-local, where O_lin-local is
 * the linear attention (ReLU feature map, the EfficientViT-style kernel the
 * page names) restricted to the same local keys.  Readings: the local keys
 * of a token are its allowed set above (same window, same wrap label, real);
 * O_lin-local uses the raw q, k (no rotation, no bias features), with
 * O_lin-local = sum_p' relu(q).relu(k_p') v_p' / sum_p' relu(q).relu(k_p'),
 * taken as 0 when that denominator is 0.
 *
 * The bias features themselves (oracle_rib_features) follow "Rank-Factorized
 * Implicit Neural Bias", section 2.1: the 2D coordinate of each window
 * position is mapped to Fourier features and a light MLP turns them into the
 * rank-r query and key factors.  Readings (the page gives no sizes):
 * coordinates c = 2 i / (M - 1) - 1 per axis (0 when M = 1); 8 octaves
 * 2^k pi, features ordered [sin(2^k pi c_y)]_k, [cos(2^k pi c_y)]_k,
 * [sin(2^k pi c_x)]_k, [cos(2^k pi c_x)]_k (32); one hidden layer of 64 with
 * tanh, no biases; separate weights per head and per side (u, w).
 *
 * The convolutional local attention gate (oracle_cla_gate) follows the same
 * page, section 2.2: a 3 x 3 depth-wise convolution and a 1 x 1 point-wise
 * convolution of the block input, a sigmoid, and the attention output
 * multiplied by that gate.  Readings: zero padding at the map border, one
 * bias per channel after each convolution, the gate applied channel by
 * channel to O of the same token.
 *
 * The backward (oracle_bwd) is the chain rule through the same steps: the
 * gradients of a scalar loss with respect to q, k, v, the RoPE frequencies
 * theta and the bias table, given the loss gradient dO at the output map.
 * The FLASHSWIN page trains the model (section "무엇과 다른가": memory was
 * what blocked training at large windows) with theta = exp(omega) learned
 * (section "어떻게 동작하나"); dL/domega = theta * dL/dtheta.  It is pinned
 * by central finite differences of the forward above.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_DTYPE_BF16 0
#define ORACLE_DTYPE_FP32 1

typedef struct {
    const void *q, *k, *v;   /* [B][H][W][heads][d], storage dtype */
    int dtype;
    const float *theta;      /* [heads][d/4] or NULL */
    const void *bias;        /* [heads][2][M*M][rank] storage dtype, or NULL */
    int B, H, W, M, shift, heads, d, rank;
    int Hp, Wp;              /* H and W rounded up to multiples of M (the padded map) */
} problem_t;

static problem_t make_problem(const void *q, const void *k, const void *v, int dtype, const float *theta,
                              const void *bias, int B, int H, int W, int M, int shift, int heads, int d,
                              int rank)
{
    problem_t p = {q, k, v, dtype, theta, bias, B, H, W, M, shift, heads, d, rank, 0, 0};
    if (M > 0) {
        p.Hp = (H + M - 1) / M * M;
        p.Wp = (W + M - 1) / M * M;
    }
    return p;
}

/* Step 1: read one stored element as fp64 (bf16 -> fp64 and fp32 -> fp64 are exact). */
static double read_elem(const void *base, int dtype, size_t idx)
{
    if (dtype == ORACLE_DTYPE_FP32)
        return (double)((const float *)base)[idx];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Step 2: the rolled map.  Rolled row yr, rolled column xr hold the padded
 * map's token at row (yr + s) mod Hp, column (xr + s) mod Wp (Hp = H and
 * Wp = W when M divides them).  Returns its element offset in the original
 * map, or -1 when that position is padding (row >= H or column >= W). */
static int64_t rolled_token_offset(const problem_t *p, int b, int yr, int xr, int h)
{
    int y = (yr + p->shift) % p->Hp;
    int x = (xr + p->shift) % p->Wp;
    if (y >= p->H || x >= p->W)
        return -1;
    return (int64_t)(((((size_t)b * p->H + y) * p->W + x) * p->heads + h) * p->d);
}

/* Step 4: window-local 2D RoPE on one d-vector at window-local (row i, col j).
 * Pair k of the first half turns by i*theta_k, pair k of the second half by
 * j*theta_k; rot(a)(x0, x1) = (x0 cos a - x1 sin a, x0 sin a + x1 cos a). */
static void rope_rotate(double *vec, int d, double i, double j, const float *theta_h)
{
    int half = d / 2;
    for (int k = 0; k < d / 4; ++k) {
        double th = (double)theta_h[k];
        double ay = i * th, ax = j * th;
        double x0 = vec[2 * k], x1 = vec[2 * k + 1];
        vec[2 * k] = x0 * cos(ay) - x1 * sin(ay);
        vec[2 * k + 1] = x0 * sin(ay) + x1 * cos(ay);
        double y0 = vec[half + 2 * k], y1 = vec[half + 2 * k + 1];
        vec[half + 2 * k] = y0 * cos(ax) - y1 * sin(ax);
        vec[half + 2 * k + 1] = y0 * sin(ax) + y1 * cos(ax);
    }
}

/* Step 6: wrap label of rolled-map row yr, column xr (0 when unshifted). */
static int wrap_label(const problem_t *p, int yr, int xr)
{
    if (p->shift == 0)
        return 0;
    return 2 * (yr >= p->Hp - p->shift) + (xr >= p->Wp - p->shift);
}

typedef struct {
    double *q, *k, *v, *s; /* N x d, N x d, N x d, N x N */
    int64_t *off;          /* N: element offset of each window token, -1 for padding */
    double *lse;           /* N: log-sum-exp of each row's masked scores (natural log) */
} scratch_t;

/* Steps 3-8 for one (batch b, window (wy, wx), head h): O = softmax(S) V in
 * window order p = i*M + j, written to out[N][d]. */
static void unit_forward(const problem_t *p, int b, int wy, int wx, int h,
                         scratch_t *w, double *out)
{
    const int M = p->M, N = M * M, d = p->d, r = p->rank;
    const double scale = 1.0 / sqrt((double)d);

    /* Step 3: gather the window's N tokens from the rolled map (a pad
     * position gets zero vectors; it is masked below and never stored). */
    for (int i = 0; i < M; ++i)
        for (int j = 0; j < M; ++j) {
            int t = i * M + j;
            int64_t off = rolled_token_offset(p, b, wy * M + i, wx * M + j, h);
            w->off[t] = off;
            for (int c = 0; c < d; ++c) {
                w->q[(size_t)t * d + c] = off < 0 ? 0.0 : read_elem(p->q, p->dtype, (size_t)off + c);
                w->k[(size_t)t * d + c] = off < 0 ? 0.0 : read_elem(p->k, p->dtype, (size_t)off + c);
                w->v[(size_t)t * d + c] = off < 0 ? 0.0 : read_elem(p->v, p->dtype, (size_t)off + c);
            }
        }

    /* Step 4: RoPE with window-local coordinates. */
    if (p->theta) {
        const float *th = p->theta + (size_t)h * (d / 4);
        for (int i = 0; i < M; ++i)
            for (int j = 0; j < M; ++j) {
                int t = i * M + j;
                rope_rotate(w->q + (size_t)t * d, d, (double)i, (double)j, th);
                rope_rotate(w->k + (size_t)t * d, d, (double)i, (double)j, th);
            }
    }

    /* Step 5: the full N x N score matrix, content scaled, bias added. */
    for (int a = 0; a < N; ++a)
        for (int c = 0; c < N; ++c) {
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += w->q[(size_t)a * d + e] * w->k[(size_t)c * d + e];
            double sc = scale * dot;
            if (p->bias) {
                size_t ub = (((size_t)h * 2 + 0) * N + a) * r;
                size_t wb = (((size_t)h * 2 + 1) * N + c) * r;
                double bd = 0.0;
                for (int e = 0; e < r; ++e)
                    bd += read_elem(p->bias, p->dtype, ub + e) * read_elem(p->bias, p->dtype, wb + e);
                sc += bd;
            }
            w->s[(size_t)a * N + c] = sc;
        }

    /* Step 6: additive -inf mask between different wrap regions, and on
     * every pad key. */
    for (int a = 0; a < N; ++a) {
        int la = wrap_label(p, wy * M + a / M, wx * M + a % M);
        for (int c = 0; c < N; ++c) {
            int lc = wrap_label(p, wy * M + c / M, wx * M + c % M);
            if (la != lc)
                w->s[(size_t)a * N + c] = -INFINITY;
            if (w->off[c] < 0)
                w->s[(size_t)a * N + c] = -INFINITY;
        }
    }

    /* Step 7: row softmax (max subtracted, exp, divided by the sum).  A pad
     * row has no output: its probabilities are zero (so nothing flows from it
     * in the backward) and step 8 marks its output NaN. */
    for (int a = 0; a < N; ++a) {
        double *row = w->s + (size_t)a * N;
        if (w->off[a] < 0) {
            for (int c = 0; c < N; ++c)
                row[c] = 0.0;
            continue;
        }
        double mx = -INFINITY;
        for (int c = 0; c < N; ++c)
            if (row[c] > mx)
                mx = row[c];
        double sum = 0.0;
        for (int c = 0; c < N; ++c) {
            row[c] = exp(row[c] - mx);
            sum += row[c];
        }
        for (int c = 0; c < N; ++c)
            row[c] /= sum;
        w->lse[a] = mx + log(sum);
    }

    /* Step 8: O = P V. */
    for (int a = 0; a < N; ++a)
        for (int e = 0; e < d; ++e) {
            double acc = 0.0;
            for (int c = 0; c < N; ++c)
                acc += w->s[(size_t)a * N + c] * w->v[(size_t)c * d + e];
            out[(size_t)a * d + e] = w->off[a] < 0 ? NAN : acc;
        }
}

/* Units are numbered u = ((b * nWy + wy) * nWx + wx) * heads + h. */
static void unit_coords(const problem_t *p, int64_t u, int *b, int *wy, int *wx, int *h)
{
    int nWy = p->Hp / p->M, nWx = p->Wp / p->M;
    *h = (int)(u % p->heads);
    u /= p->heads;
    *wx = (int)(u % nWx);
    u /= nWx;
    *wy = (int)(u % nWy);
    *b = (int)(u / nWy);
}

typedef struct {
    const problem_t *p;
    const int64_t *units;  /* NULL = every unit in order */
    int64_t n_units;
    double *out_units;     /* [n_units][N][d] or NULL */
    double *out_map;       /* [B][H][W][heads][d] or NULL (step 9 scatter) */
    double *lse_map;       /* [B][H][W][heads] or NULL: each row's log-sum-exp, scattered like O */
    int64_t next;          /* shared work counter */
    int failed;
} job_t;

static void *worker(void *arg)
{
    job_t *job = (job_t *)arg;
    const problem_t *p = job->p;
    const size_t N = (size_t)p->M * p->M, d = (size_t)p->d;
    scratch_t w;
    w.q = malloc(N * d * sizeof(double));
    w.k = malloc(N * d * sizeof(double));
    w.v = malloc(N * d * sizeof(double));
    w.s = malloc(N * N * sizeof(double));
    w.off = malloc(N * sizeof(int64_t));
    w.lse = malloc(N * sizeof(double));
    double *o = malloc(N * d * sizeof(double));
    if (!w.q || !w.k || !w.v || !w.s || !w.off || !w.lse || !o) {
        __atomic_store_n(&job->failed, 1, __ATOMIC_RELAXED);
        goto done;
    }
    for (;;) {
        int64_t n = __atomic_fetch_add(&job->next, 1, __ATOMIC_RELAXED);
        if (n >= job->n_units)
            break;
        int64_t u = job->units ? job->units[n] : n;
        int b, wy, wx, h;
        unit_coords(p, u, &b, &wy, &wx, &h);
        double *dst = job->out_units ? job->out_units + (size_t)n * N * d : o;
        unit_forward(p, b, wy, wx, h, &w, dst);
        if (job->out_map) {
            /* Step 9: write back through the inverse roll, i.e. to the same
             * original position each token was gathered from (pads: nowhere). */
            for (int i = 0; i < p->M; ++i)
                for (int j = 0; j < p->M; ++j) {
                    int64_t off = rolled_token_offset(p, b, wy * p->M + i, wx * p->M + j, h);
                    if (off >= 0) {
                        memcpy(job->out_map + off, dst + ((size_t)i * p->M + j) * d, d * sizeof(double));
                        if (job->lse_map)
                            job->lse_map[off / (int64_t)d] = w.lse[i * p->M + j];
                    }
                }
        }
    }
done:
    free(w.q);
    free(w.k);
    free(w.v);
    free(w.s);
    free(w.off);
    free(w.lse);
    free(o);
    return NULL;
}

static int check_problem(const problem_t *p)
{
    if (!p->q || !p->k || !p->v)
        return -1;
    if (p->dtype != ORACLE_DTYPE_BF16 && p->dtype != ORACLE_DTYPE_FP32)
        return -1;
    if (p->B <= 0 || p->H <= 0 || p->W <= 0 || p->M <= 0 || p->heads <= 0)
        return -1;
    if (p->shift < 0 || p->shift >= p->M)
        return -1;
    if (p->d <= 0 || p->d % 4)
        return -1;
    if ((p->rank > 0) != (p->bias != NULL) || p->rank < 0)
        return -1;
    return 0;
}

static int run(const problem_t *p, const int64_t *units, int64_t n_units,
               double *out_units, double *out_map, double *lse_map, int nthreads, double mem_budget_bytes)
{
    if (check_problem(p))
        return -1;
    if (n_units <= 0)
        return 0;
    long ncpu = sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads <= 0)
        nthreads = ncpu > 0 ? (int)ncpu : 1;
    double per_thread = ((double)p->M * p->M) * ((double)p->M * p->M + 4.0 * p->d) * sizeof(double);
    if (mem_budget_bytes <= 0)
        mem_budget_bytes = 8e9;
    int cap = (int)(mem_budget_bytes / per_thread);
    if (cap < 1)
        cap = 1;
    if (nthreads > cap)
        nthreads = cap;
    if (nthreads > n_units)
        nthreads = (int)n_units;

    job_t job = {p, units, n_units, out_units, out_map, lse_map, 0, 0};
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th)
        return -2;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, worker, &job) != 0)
            break;
        ++started;
    }
    if (started == 0)
        worker(&job);
    for (int t = 0; t < started; ++t)
        pthread_join(th[t], NULL);
    free(th);
    return job.failed ? -2 : (started == 0 ? 1 : started);
}

/* ---- exported entry points (called through ctypes by oracle/__init__.py) ---- */

/* Every unit; output scattered to out_map [B][H][W][heads][d] fp64.
 * Returns the number of threads used (> 0), or < 0 on bad arguments. */
int oracle_fwd(const void *q, const void *k, const void *v, int dtype,
               const float *theta, const void *bias,
               int B, int H, int W, int M, int shift, int heads, int d, int rank,
               double *out_map, int nthreads, double mem_budget_bytes)
{
    problem_t p = make_problem(q, k, v, dtype, theta, bias, B, H, W, M, shift, heads, d, rank);
    if (check_problem(&p) || !out_map)
        return -1;
    int64_t n = (int64_t)B * (p.Hp / M) * (p.Wp / M) * heads;
    return run(&p, NULL, n, NULL, out_map, NULL, nthreads, mem_budget_bytes);
}

/* As oracle_fwd, and also each row's log-sum-exp (natural log of the sum of
 * exp of its masked scores, z = d^-1/2 q.k + u.w) into lse_map
 * [B][H][W][heads] fp64. */
int oracle_fwd_lse(const void *q, const void *k, const void *v, int dtype,
                   const float *theta, const void *bias,
                   int B, int H, int W, int M, int shift, int heads, int d, int rank,
                   double *out_map, double *lse_map, int nthreads, double mem_budget_bytes)
{
    problem_t p = make_problem(q, k, v, dtype, theta, bias, B, H, W, M, shift, heads, d, rank);
    if (check_problem(&p) || !out_map || !lse_map)
        return -1;
    int64_t n = (int64_t)B * (p.Hp / M) * (p.Wp / M) * heads;
    return run(&p, NULL, n, NULL, out_map, lse_map, nthreads, mem_budget_bytes);
}

/* Selected units; out_units [n_units][M*M][d] fp64 in window order p = i*M + j
 * (NaN rows at pad positions). */
int oracle_fwd_units(const void *q, const void *k, const void *v, int dtype,
                     const float *theta, const void *bias,
                     int B, int H, int W, int M, int shift, int heads, int d, int rank,
                     const int64_t *units, int64_t n_units,
                     double *out_units, int nthreads, double mem_budget_bytes)
{
    problem_t p = make_problem(q, k, v, dtype, theta, bias, B, H, W, M, shift, heads, d, rank);
    if (check_problem(&p) || !units || !out_units)
        return -1;
    int64_t total = (int64_t)B * (p.Hp / M) * (p.Wp / M) * heads;
    for (int64_t n = 0; n < n_units; ++n)
        if (units[n] < 0 || units[n] >= total)
            return -1;
    return run(&p, units, n_units, out_units, NULL, NULL, nthreads, mem_budget_bytes);
}

/* The gated residual: out_map [B][H][W][heads][d] fp64 holds O_lin on entry;
 * for every token of each listed window w = (b * nWy + wy) * nWx + wx (all
 * heads), out += O_local - O_lin-local.  Windows may not repeat.  Plain
 * loops, one window-head at a time. */
int oracle_fwd_sparse(const void *q, const void *k, const void *v, int dtype,
                      const float *theta, const void *bias,
                      int B, int H, int W, int M, int shift, int heads, int d, int rank,
                      const int32_t *windows, int64_t n_windows, double *out_map)
{
    problem_t p = make_problem(q, k, v, dtype, theta, bias, B, H, W, M, shift, heads, d, rank);
    if (check_problem(&p) || !out_map || (n_windows > 0 && !windows) || d > 256)
        return -1;
    const int nWy = p.Hp / M, nWx = p.Wp / M;
    const int64_t total = (int64_t)B * nWy * nWx;
    for (int64_t n = 0; n < n_windows; ++n)
        if (windows[n] < 0 || windows[n] >= total)
            return -1;
    const size_t N = (size_t)M * M;
    scratch_t w;
    w.q = malloc(N * d * sizeof(double));
    w.k = malloc(N * d * sizeof(double));
    w.v = malloc(N * d * sizeof(double));
    w.s = malloc(N * N * sizeof(double));
    w.off = malloc(N * sizeof(int64_t));
    w.lse = malloc(N * sizeof(double));
    double *o = malloc(N * d * sizeof(double));
    double *kq = malloc(N * (size_t)d * 2 * sizeof(double));  /* relu(q), relu(k) of the raw rows */
    int rc = 0;
    if (!w.q || !w.k || !w.v || !w.s || !w.off || !w.lse || !o || !kq) {
        rc = -2;
        goto done;
    }
    for (int64_t n = 0; n < n_windows; ++n) {
        const int wid = windows[n];
        const int b = wid / (nWy * nWx), wy = (wid / nWx) % nWy, wx = wid % nWx;
        for (int h = 0; h < heads; ++h) {
            unit_forward(&p, b, wy, wx, h, &w, o);
            /* the raw rows (unit_forward rotated q, k in place): re-read */
            for (size_t t = 0; t < N; ++t)
                for (int c = 0; c < d; ++c) {
                    const int64_t off = w.off[t];
                    const double qr = off < 0 ? 0.0 : read_elem(p.q, p.dtype, (size_t)off + c);
                    const double kr = off < 0 ? 0.0 : read_elem(p.k, p.dtype, (size_t)off + c);
                    kq[t * d + c] = qr > 0.0 ? qr : 0.0;
                    kq[(N + t) * d + c] = kr > 0.0 ? kr : 0.0;
                }
            for (size_t a = 0; a < N; ++a) {
                if (w.off[a] < 0)
                    continue;
                const int la = wrap_label(&p, wy * M + (int)a / M, wx * M + (int)a % M);
                double den = 0.0;
                double num[256];
                for (int e = 0; e < d; ++e)
                    num[e] = 0.0;
                for (size_t c = 0; c < N; ++c) {
                    if (w.off[c] < 0 || wrap_label(&p, wy * M + (int)c / M, wx * M + (int)c % M) != la)
                        continue;
                    double wgt = 0.0;
                    for (int e = 0; e < d; ++e)
                        wgt += kq[a * d + e] * kq[(N + c) * d + e];
                    den += wgt;
                    for (int e = 0; e < d; ++e)
                        num[e] += wgt * w.v[c * d + e];
                }
                double *dst = out_map + w.off[a];
                for (int e = 0; e < d; ++e)
                    dst[e] += o[a * d + e] - (den > 0.0 ? num[e] / den : 0.0);
            }
        }
    }
done:
    free(w.q);
    free(w.k);
    free(w.v);
    free(w.s);
    free(w.off);
    free(w.lse);
    free(o);
    free(kq);
    return rc;
}

/* The rank-r factor table [heads][2][M*M][rank] (fp64) from the MLP weights
 * w1 [heads][2][32][64] and w2 [heads][2][64][rank] (fp32). */
int oracle_rib_features(const float *w1, const float *w2, int M, int heads, int rank, double *table)
{
    if (!w1 || !w2 || !table || M <= 0 || heads <= 0 || rank <= 0)
        return -1;
    const int N = M * M;
    for (int h = 0; h < heads; ++h)
        for (int side = 0; side < 2; ++side) {
            const float *a = w1 + ((size_t)h * 2 + side) * 32 * 64;
            const float *b = w2 + ((size_t)h * 2 + side) * 64 * rank;
            for (int p = 0; p < N; ++p) {
                const int i = p / M, j = p % M;
                /* Fourier features of the window-local coordinate */
                const double cy = M > 1 ? 2.0 * i / (M - 1) - 1.0 : 0.0;
                const double cx = M > 1 ? 2.0 * j / (M - 1) - 1.0 : 0.0;
                double f[32];
                for (int k = 0; k < 8; ++k) {
                    const double w = ldexp(acos(-1.0), k);  /* 2^k pi */
                    f[k] = sin(w * cy);
                    f[8 + k] = cos(w * cy);
                    f[16 + k] = sin(w * cx);
                    f[24 + k] = cos(w * cx);
                }
                /* the MLP: tanh(f w1) w2 */
                double hid[64];
                for (int c = 0; c < 64; ++c) {
                    double acc = 0.0;
                    for (int e = 0; e < 32; ++e)
                        acc += f[e] * a[e * 64 + c];
                    hid[c] = tanh(acc);
                }
                double *dst = table + (((size_t)h * 2 + side) * N + p) * rank;
                for (int r = 0; r < rank; ++r) {
                    double acc = 0.0;
                    for (int c = 0; c < 64; ++c)
                        acc += hid[c] * b[c * rank + r];
                    dst[r] = acc;
                }
            }
        }
    return 0;
}

/* The gated attention output: out = O * sigmoid(PW(DW3x3(x))), all
 * [B][H][W][C] fp64 (x and O as read from their storage dtype), dw
 * [C][3][3], dw_b [C], pw [C_out][C_in], pw_b [C] fp32. */
int oracle_cla_gate(const void *x, const void *o, int dtype, const float *dw, const float *dw_b, const float *pw,
                    const float *pw_b, int B, int H, int W, int C, double *out)
{
    if (!x || !o || !dw || !dw_b || !pw || !pw_b || !out || B <= 0 || H <= 0 || W <= 0 || C <= 0)
        return -1;
    double *y = malloc((size_t)C * sizeof(double));
    if (!y)
        return -2;
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < H; ++r)
            for (int c = 0; c < W; ++c) {
                /* depth-wise 3 x 3, zero outside the map */
                for (int ch = 0; ch < C; ++ch) {
                    double acc = dw_b[ch];
                    for (int dy = -1; dy <= 1; ++dy)
                        for (int dx = -1; dx <= 1; ++dx) {
                            const int rr = r + dy, cc = c + dx;
                            if (rr < 0 || rr >= H || cc < 0 || cc >= W)
                                continue;
                            acc += dw[ch * 9 + (dy + 1) * 3 + (dx + 1)] *
                                   read_elem(x, dtype, (((size_t)b * H + rr) * W + cc) * C + ch);
                        }
                    y[ch] = acc;
                }
                /* point-wise 1 x 1, sigmoid, gate */
                for (int co = 0; co < C; ++co) {
                    double acc = pw_b[co];
                    for (int ci = 0; ci < C; ++ci)
                        acc += pw[(size_t)co * C + ci] * y[ci];
                    const size_t idx = (((size_t)b * H + r) * W + c) * C + co;
                    out[idx] = read_elem(o, dtype, idx) / (1.0 + exp(-acc));
                }
            }
    free(y);
    return 0;
}

/* The rotation alone, for the displacement-identity checks: out = R(i, j) vec. */
int oracle_rope(const double *vec, int d, double i, double j, const float *theta_h, double *out)
{
    if (!vec || !theta_h || !out || d <= 0 || d % 4)
        return -1;
    memcpy(out, vec, (size_t)d * sizeof(double));
    rope_rotate(out, d, i, j, theta_h);
    return 0;
}

/* Original (row, col) of rolled-window token p of window (wy, wx), in the
 * padded map; returns 1 when that position is padding, 0 for a real token. */
int oracle_token_origin(int H, int W, int M, int shift, int wy, int wx, int p, int *y, int *x)
{
    if (M <= 0 || p < 0 || p >= M * M || !y || !x)
        return -1;
    const int Hp = (H + M - 1) / M * M, Wp = (W + M - 1) / M * M;
    *y = (wy * M + p / M + shift) % Hp;
    *x = (wx * M + p % M + shift) % Wp;
    return (*y >= H || *x >= W) ? 1 : 0;
}

/* ---- backward ---------------------------------------------------------------
 * For one unit, after unit_forward has left the rotated q~, k~, v and the
 * probabilities P in the scratch, with dO the loss gradient at the unit's
 * output rows (gathered from the same original positions):
 *   dV[c]    = sum_a P[a][c] dO[a]
 *   dP[a][c] = dO[a] . v[c]
 *   dS[a][c] = P[a][c] (dP[a][c] - sum_c' P[a][c'] dP[a][c'])
 *   dq~[a] = scale sum_c dS[a][c] k~[c],   dk~[c] = scale sum_a dS[a][c] q~[a]
 *   du[a]  = sum_c dS[a][c] w[c],          dw[c]  = sum_a dS[a][c] u[a]
 *   dq = R(i, j)^T dq~ = R(-i, -j) dq~,    dk likewise
 *   dtheta_k += i (dx~_{2k+1} x~_{2k} - dx~_{2k} x~_{2k+1})
 *             + j (dx~_{h+2k+1} x~_{h+2k} - dx~_{h+2k} x~_{h+2k+1})  for x = q and k, h = d/2
 * (d/dtheta of the pair rotation by angle i*theta maps (x~0, x~1) to
 * i (-x~1, x~0)).  Every token lies in exactly one window of a call, so dq,
 * dk, dv are written, not accumulated; dtheta and the bias-table gradient sum
 * over all windows and images of a head. */

typedef struct {
    const problem_t *p;
    const double *dout;
    double *dq, *dk, *dv;   /* maps like dout */
    double *dtheta;         /* [heads][d/4] or NULL */
    double *dbias;          /* [heads][2][N][rank] or NULL */
    int64_t n_units;
    int64_t next;
    int failed;
    pthread_mutex_t mu;
} bwd_job_t;

static void unit_backward(const problem_t *p, int b, int wy, int wx, int h, const scratch_t *w,
                          const double *dout, double *dq, double *dk, double *dv,
                          double *dtheta_h, double *dbias_h, double *g_o, double *g_s, double *g_q, double *g_k)
{
    const int M = p->M, N = M * M, d = p->d, r = p->rank;
    const double scale = 1.0 / sqrt((double)p->d);  /* the forward's d^-1/2 */

    /* dO of the unit's rows, from the tokens' original positions (zero at
     * pad rows, which have no output) */
    for (int t = 0; t < N; ++t) {
        if (w->off[t] < 0)
            memset(g_o + (size_t)t * d, 0, (size_t)d * sizeof(double));
        else
            memcpy(g_o + (size_t)t * d, dout + w->off[t], (size_t)d * sizeof(double));
    }
    /* dV, scattered straight to the map */
    for (int c = 0; c < N; ++c) {
        const int64_t off = w->off[c];
        if (off < 0)
            continue;
        for (int e = 0; e < d; ++e) {
            double acc = 0.0;
            for (int a = 0; a < N; ++a)
                acc += w->s[(size_t)a * N + c] * g_o[(size_t)a * d + e];
            dv[off + e] = acc;
        }
    }
    /* dP, then dS in place */
    for (int a = 0; a < N; ++a) {
        double rowdot = 0.0;
        for (int c = 0; c < N; ++c) {
            double dp = 0.0;
            for (int e = 0; e < d; ++e)
                dp += g_o[(size_t)a * d + e] * w->v[(size_t)c * d + e];
            g_s[(size_t)a * N + c] = dp;
            rowdot += w->s[(size_t)a * N + c] * dp;
        }
        for (int c = 0; c < N; ++c)
            g_s[(size_t)a * N + c] = w->s[(size_t)a * N + c] * (g_s[(size_t)a * N + c] - rowdot);
    }
    /* dq~, dk~ */
    for (int a = 0; a < N; ++a)
        for (int e = 0; e < d; ++e) {
            double acc = 0.0;
            for (int c = 0; c < N; ++c)
                acc += g_s[(size_t)a * N + c] * w->k[(size_t)c * d + e];
            g_q[(size_t)a * d + e] = scale * acc;
        }
    for (int c = 0; c < N; ++c)
        for (int e = 0; e < d; ++e) {
            double acc = 0.0;
            for (int a = 0; a < N; ++a)
                acc += g_s[(size_t)a * N + c] * w->q[(size_t)a * d + e];
            g_k[(size_t)c * d + e] = scale * acc;
        }
    /* bias-table gradient: du (side 0, query rows) and dw (side 1, key rows) */
    if (p->bias && dbias_h) {
        for (int a = 0; a < N; ++a)
            for (int e = 0; e < r; ++e) {
                double acc = 0.0;
                for (int c = 0; c < N; ++c)
                    acc += g_s[(size_t)a * N + c] * read_elem(p->bias, p->dtype, (((size_t)h * 2 + 1) * N + c) * r + e);
                dbias_h[(size_t)a * r + e] += acc;
            }
        for (int c = 0; c < N; ++c)
            for (int e = 0; e < r; ++e) {
                double acc = 0.0;
                for (int a = 0; a < N; ++a)
                    acc += g_s[(size_t)a * N + c] * read_elem(p->bias, p->dtype, (((size_t)h * 2 + 0) * N + a) * r + e);
                dbias_h[((size_t)N + c) * r + e] += acc;
            }
    }
    /* theta gradient, then back through the rotation */
    const int half = d / 2;
    for (int t = 0; t < N; ++t) {
        const double i = (double)(t / M), j = (double)(t % M);
        double *gq = g_q + (size_t)t * d, *gk = g_k + (size_t)t * d;
        const double *xq = w->q + (size_t)t * d, *xk = w->k + (size_t)t * d;
        if (p->theta) {
            if (dtheta_h)
                for (int k = 0; k < d / 4; ++k) {
                    const int a0 = 2 * k, a1 = 2 * k + 1, b0 = half + 2 * k, b1 = half + 2 * k + 1;
                    dtheta_h[k] += i * (gq[a1] * xq[a0] - gq[a0] * xq[a1]) + j * (gq[b1] * xq[b0] - gq[b0] * xq[b1]) +
                                   i * (gk[a1] * xk[a0] - gk[a0] * xk[a1]) + j * (gk[b1] * xk[b0] - gk[b0] * xk[b1]);
                }
            const float *th = p->theta + (size_t)h * (d / 4);
            rope_rotate(gq, d, -i, -j, th);
            rope_rotate(gk, d, -i, -j, th);
        }
        if (w->off[t] >= 0) {
            memcpy(dq + w->off[t], gq, (size_t)d * sizeof(double));
            memcpy(dk + w->off[t], gk, (size_t)d * sizeof(double));
        }
    }
}

static void *bwd_worker(void *arg)
{
    bwd_job_t *job = (bwd_job_t *)arg;
    const problem_t *p = job->p;
    const size_t N = (size_t)p->M * p->M, d = (size_t)p->d, r = (size_t)p->rank;
    const size_t nth = (size_t)p->heads * (d / 4), nbias = (size_t)p->heads * 2 * N * r;
    scratch_t w;
    w.q = malloc(N * d * sizeof(double));
    w.k = malloc(N * d * sizeof(double));
    w.v = malloc(N * d * sizeof(double));
    w.s = malloc(N * N * sizeof(double));
    w.off = malloc(N * sizeof(int64_t));
    w.lse = malloc(N * sizeof(double));
    double *o = malloc(N * d * sizeof(double));
    double *g_o = malloc(N * d * sizeof(double)), *g_s = malloc(N * N * sizeof(double));
    double *g_q = malloc(N * d * sizeof(double)), *g_k = malloc(N * d * sizeof(double));
    double *dth = job->dtheta ? calloc(nth, sizeof(double)) : NULL;
    double *dbi = job->dbias ? calloc(nbias > 0 ? nbias : 1, sizeof(double)) : NULL;
    if (!w.q || !w.k || !w.v || !w.s || !w.off || !w.lse || !o || !g_o || !g_s || !g_q || !g_k || (job->dtheta && !dth) ||
        (job->dbias && !dbi)) {
        __atomic_store_n(&job->failed, 1, __ATOMIC_RELAXED);
        goto done;
    }
    for (;;) {
        int64_t n = __atomic_fetch_add(&job->next, 1, __ATOMIC_RELAXED);
        if (n >= job->n_units)
            break;
        int b, wy, wx, h;
        unit_coords(p, n, &b, &wy, &wx, &h);
        unit_forward(p, b, wy, wx, h, &w, o);
        unit_backward(p, b, wy, wx, h, &w, job->dout, job->dq, job->dk, job->dv,
                      dth ? dth + (size_t)h * (d / 4) : NULL, dbi ? dbi + (size_t)h * 2 * N * r : NULL,
                      g_o, g_s, g_q, g_k);
    }
    pthread_mutex_lock(&job->mu);
    if (dth)
        for (size_t e = 0; e < nth; ++e)
            job->dtheta[e] += dth[e];
    if (dbi)
        for (size_t e = 0; e < nbias; ++e)
            job->dbias[e] += dbi[e];
    pthread_mutex_unlock(&job->mu);
done:
    free(w.q);
    free(w.k);
    free(w.v);
    free(w.s);
    free(w.off);
    free(w.lse);
    free(o);
    free(g_o);
    free(g_s);
    free(g_q);
    free(g_k);
    free(dth);
    free(dbi);
    return NULL;
}

/* Gradients of a scalar loss L given dout = dL/dO [B][H][W][heads][d] (fp64):
 * dq, dk, dv in the same layout, dtheta [heads][d/4] (NULL without theta),
 * dbias [heads][2][M*M][rank] (NULL without bias), all fp64 and overwritten.
 * Returns the number of threads used (> 0), or < 0 on bad arguments. */
int oracle_bwd(const void *q, const void *k, const void *v, int dtype,
               const float *theta, const void *bias,
               int B, int H, int W, int M, int shift, int heads, int d, int rank,
               const double *dout, double *dq, double *dk, double *dv, double *dtheta, double *dbias,
               int nthreads)
{
    problem_t p = make_problem(q, k, v, dtype, theta, bias, B, H, W, M, shift, heads, d, rank);
    if (check_problem(&p) || !dout || !dq || !dk || !dv)
        return -1;
    if ((dtheta != NULL && theta == NULL) || (dbias != NULL && bias == NULL))
        return -1;
    const size_t N = (size_t)M * M;
    if (dtheta)
        memset(dtheta, 0, (size_t)heads * (d / 4) * sizeof(double));
    if (dbias)
        memset(dbias, 0, (size_t)heads * 2 * N * rank * sizeof(double));
    int64_t n_units = (int64_t)B * (p.Hp / M) * (p.Wp / M) * heads;
    long ncpu = sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads <= 0)
        nthreads = ncpu > 0 ? (int)ncpu : 1;
    if (nthreads > n_units)
        nthreads = (int)n_units;
    bwd_job_t job;
    memset(&job, 0, sizeof job);
    job.p = &p;
    job.dout = dout;
    job.dq = dq;
    job.dk = dk;
    job.dv = dv;
    job.dtheta = dtheta;
    job.dbias = dbias;
    job.n_units = n_units;
    pthread_mutex_init(&job.mu, NULL);
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) {
        pthread_mutex_destroy(&job.mu);
        return -2;
    }
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, bwd_worker, &job) != 0)
            break;
        ++started;
    }
    if (started == 0)
        bwd_worker(&job);
    for (int t = 0; t < started; ++t)
        pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&job.mu);
    return job.failed ? -2 : (started == 0 ? 1 : started);
}
