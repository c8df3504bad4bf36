/*
 * Plain fp64 CPU oracle for causal scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may link, load or call this file; only the tests, the
 * smoke check and the CPU-baseline leg of the benchmark do.  It shares no code
 * with the CUDA kernels: it is a slow, literal restatement of the definition.
 *
 * What it computes, for every requested output row (b, h, i):
 *
 *   g    = H / Hkv, kvh = floor(h / g)          grouped-query head mapping
 *        ("Grouped-Query Attention" §5.1: each K/V head is copied group_size
 *         times with repeat_interleave, so query head h reads K/V head h / g;
 *         "Hesper.Layers.Attention" reshapeToHeadsKernel: kv_head = oh / headsPerKVHead)
 *   p    = start_pos + i                          absolute position of query i
 *        ("makarna attention_cached.go" CausalAttentionCached: new tokens start
 *         at startPos, the history holds every earlier and current key)
 *   vis  = { j < S : (!causal or j <= p) and (window = 0 or j > p - window) }
 *        causal mask: 0 on and below the diagonal, -inf above
 *        ("Hesper.Layers.Attention" Causal Masking; "Grouped-Query Attention"
 *        §5.2); a local window of w keys keeps only the current position and
 *        the previous w - 1 ("Multi-query attention, annotated" §4.1: local
 *        versions attend to the current position and the previous 31)
 *   s_j  = scale * sum_t Q[b,h,i,t] * K[b,kvh,j,t]   for j in vis
 *        (scores = Q K^T / sqrt(d_k): "Hesper.Layers.Attention" Mathematical
 *         Definition; the scale is an explicit argument because the worked
 *         example of "Multi-query attention, annotated" §2.1 is unscaled)
 *   M    = max_j s_j,  w_j = exp(s_j - M),  L = sum_j w_j     (two-pass softmax,
 *        materialised, not online: "Causal Multi-Head Self-Attention" —
 *        Two exact full-sequence algorithms, the materialized one)
 *   O    = sum_j (w_j / L) * V[b,kvh,j,:]          masked j contribute nothing
 *   lse  = M + ln L,   prob_j = w_j / L  (0 for masked j)
 *
 * Inputs are widened exactly to double: fp32 by C conversion, bf16 and fp16 by
 * the bit-level conversions below (both exact by construction).  All sums are
 * plain left-to-right double accumulation; no blocking, no reordering.
 *
 * Every function here is pinned by CPU tests against values that do not come
 * from this file: the worked example printed on the "Multi-query attention,
 * annotated" page, closed forms, invariants, an exhaustive check of the
 * widening against library conversions, and an independent library routine.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F16 = 2, ORACLE_F64 = 3 };

/* bf16 is the upper half of an IEEE binary32: shifting its 16 bits into the
 * top of a 32-bit word gives the binary32 with the same value. */
double oracle_widen_bf16(uint16_t bits) {
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Normal: (-1)^s * (1024 + frac) * 2^(e - 25); subnormal: frac * 2^-24. */
double oracle_widen_f16(uint16_t bits) {
    int sign = (bits >> 15) & 1;
    int e = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double mag;
    if (e == 0x1f) {
        mag = frac ? NAN : INFINITY;
    } else if (e == 0) {
        mag = ldexp((double)frac, -24);
    } else {
        mag = ldexp((double)(1024 + frac), e - 25);
    }
    return sign ? -mag : mag;
}

static double load_elem(const void* base, int dtype, int64_t idx) {
    switch (dtype) {
    case ORACLE_F32: return (double)((const float*)base)[idx];
    case ORACLE_BF16: return oracle_widen_bf16(((const uint16_t*)base)[idx]);
    case ORACLE_F16: return oracle_widen_f16(((const uint16_t*)base)[idx]);
    default: return ((const double*)base)[idx];
    }
}

typedef struct {
    const void *q, *k, *v;
    int dtype;
    int64_t B, H, Hkv, Tq, S, S_cap, d, start_pos;
    double scale;
    int causal;
    int64_t window; /* 0: no window */
    const int64_t* rows;
    int64_t nrows;
    double *out, *lse, *probs;
    int64_t first, last; /* half-open range of requested rows for one worker */
    int status;
} job_t;

/* Is key j visible to the query at absolute position p? */
static int visible(const job_t* J, int64_t j, int64_t p) {
    if (J->causal && j > p) return 0;
    if (J->window > 0 && j <= p - J->window) return 0;
    return 1;
}

/* One output row, straight from the definition in the file header. */
static int one_row(const job_t* J, int64_t slot, double* s, double* w) {
    int64_t r = J->rows ? J->rows[slot] : slot;
    int64_t i = r % J->Tq;
    int64_t h = (r / J->Tq) % J->H;
    int64_t b = r / (J->Tq * J->H);
    int64_t g = J->H / J->Hkv;
    int64_t kvh = h / g;
    int64_t p = J->start_pos + i;
    int64_t d = J->d;
    int64_t q_off = ((b * J->H + h) * J->Tq + i) * d;
    int64_t kv_base = (b * J->Hkv + kvh) * J->S_cap;
    double* o = J->out + slot * d;

    /* visible keys and their scores */
    int64_t nvis = 0;
    for (int64_t j = 0; j < J->S; ++j) {
        if (!visible(J, j, p)) continue;
        double dot = 0.0;
        for (int64_t t = 0; t < d; ++t)
            dot += load_elem(J->q, J->dtype, q_off + t) *
                   load_elem(J->k, J->dtype, (kv_base + j) * d + t);
        s[j] = J->scale * dot;
        ++nvis;
    }
    for (int64_t t = 0; t < d; ++t) o[t] = 0.0;
    if (J->probs)
        for (int64_t j = 0; j < J->S; ++j) J->probs[slot * J->S + j] = 0.0;
    if (nvis == 0) {
        /* A row that sees no key has an empty softmax; it is reported as zeros
         * (the makarna CPU loop leaves such a row at zero).  The CUDA library
         * rejects the arguments that would produce one. */
        if (J->lse) J->lse[slot] = -INFINITY;
        return 0;
    }

    /* pass 1: maximum over the visible scores */
    double M = -INFINITY;
    for (int64_t j = 0; j < J->S; ++j) {
        if (!visible(J, j, p)) continue;
        if (s[j] > M) M = s[j];
    }
    /* pass 2: exponentials and their sum */
    double L = 0.0;
    for (int64_t j = 0; j < J->S; ++j) {
        if (!visible(J, j, p)) { w[j] = 0.0; continue; }
        w[j] = exp(s[j] - M);
        L += w[j];
    }
    /* weighted sum of the visible value rows */
    for (int64_t j = 0; j < J->S; ++j) {
        if (!visible(J, j, p)) continue;
        double pj = w[j] / L;
        if (J->probs) J->probs[slot * J->S + j] = pj;
        for (int64_t t = 0; t < d; ++t)
            o[t] += pj * load_elem(J->v, J->dtype, (kv_base + j) * d + t);
    }
    if (J->lse) J->lse[slot] = M + log(L);
    return 0;
}

static void* worker(void* arg) {
    job_t* J = (job_t*)arg;
    double* s = (double*)malloc(sizeof(double) * (size_t)(J->S > 0 ? J->S : 1));
    double* w = (double*)malloc(sizeof(double) * (size_t)(J->S > 0 ? J->S : 1));
    if (!s || !w) { J->status = -2; free(s); free(w); return NULL; }
    for (int64_t slot = J->first; slot < J->last; ++slot) one_row(J, slot, s, w);
    free(s);
    free(w);
    return NULL;
}

/*
 * q: [B, H, Tq, d]; k, v: [B, Hkv, S_cap, d] with the first S rows valid.
 * rows: optional list of flat row ids ((b*H + h)*Tq + i); NULL means every row
 * in order.  out: [nrows, d]; lse: nullable [nrows]; probs: nullable [nrows, S].
 * nthreads <= 0 uses every online core.  Returns 0, or a negative code on a
 * malformed argument (checked here so the tests can rely on it).
 */
int oracle_attention_window(const void* q, const void* k, const void* v, int dtype,
                            int64_t B, int64_t H, int64_t Hkv, int64_t Tq, int64_t S,
                            int64_t S_cap, int64_t d, int64_t start_pos, double scale,
                            int causal, int64_t window, const int64_t* rows, int64_t nrows,
                            double* out, double* lse, double* probs, int nthreads) {
    if (B < 0 || H <= 0 || Hkv <= 0 || H % Hkv || Tq < 0 || S < 0 || S_cap < S ||
        d <= 0 || start_pos < 0 || dtype < 0 || dtype > 3 || window < 0)
        return -1;
    int64_t total = B * H * Tq;
    if (!rows) nrows = total;
    if (rows)
        for (int64_t n = 0; n < nrows; ++n)
            if (rows[n] < 0 || rows[n] >= total) return -1;
    if (nrows == 0) return 0;

    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nrows) nthreads = (int)nrows;

    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return -2; }
    int status = 0;
    for (int t = 0; t < nthreads; ++t) {
        job_t* J = &jobs[t];
        J->q = q; J->k = k; J->v = v; J->dtype = dtype;
        J->B = B; J->H = H; J->Hkv = Hkv; J->Tq = Tq; J->S = S; J->S_cap = S_cap;
        J->d = d; J->start_pos = start_pos; J->scale = scale; J->causal = causal;
        J->window = window;
        J->rows = rows; J->nrows = nrows; J->out = out; J->lse = lse; J->probs = probs;
        J->first = nrows * t / nthreads;
        J->last = nrows * (t + 1) / nthreads;
        if (nthreads == 1) {
            worker(J);
        } else if (pthread_create(&tid[t], NULL, worker, J) != 0) {
            worker(J); /* run inline if a thread cannot be created */
            tid[t] = 0;
        }
    }
    if (nthreads > 1)
        for (int t = 0; t < nthreads; ++t)
            if (tid[t]) pthread_join(tid[t], NULL);
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].status) status = jobs[t].status;
    free(jobs);
    free(tid);
    return status;
}

int oracle_num_cores(void) { return (int)sysconf(_SC_NPROCESSORS_ONLN); }

/*
 * KV-cache append with rotary position embedding on K (NeoX pairing).
 *
 * Follows "Hesper.Layers.Attention", fusedRopeKAndCacheWriteKernel (RoPE on
 * the new K, written together with V into the cache slot at the token's
 * position; the rotation partner of dimension i < d/2 is i + d/2) and
 * kvWriteBatchKernelF16 (the same write without rotation), and "Grouped-Query
 * Attention" §5.1 (apply_rope with offset = start_pos before the cache
 * append).  The frequency of pair i is base^(-2i/d) — the pages leave that
 * formula unrendered; this is the reading stated in the design notes.
 *
 * For every b < B, kv head h < Hkv, new token t < Tnew at position
 * p = start_pos + t, and i < d/2 with a = p * base^(-2i/d):
 *   K_out[i]       = K[i] cos a - K[i + d/2] sin a
 *   K_out[i + d/2] = K[i + d/2] cos a + K[i] sin a
 *   V_out          = V
 * base <= 0 means no rotation.  Inputs k_new, v_new: [B, Hkv, Tnew, d];
 * outputs (fp64) k_out, v_out: [B, Hkv, Tnew, d] (the rows to be written at
 * positions start_pos .. start_pos + Tnew - 1).
 */
int oracle_rope_append(const void* k_new, const void* v_new, int dtype, int64_t B, int64_t Hkv,
                       int64_t Tnew, int64_t d, int64_t start_pos, double base, double* k_out,
                       double* v_out) {
    if (B < 0 || Hkv < 0 || Tnew < 0 || d <= 0 || (d & 1) || start_pos < 0 || dtype < 0 ||
        dtype > 3)
        return -1;
    const int64_t h = d / 2;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t kv = 0; kv < Hkv; ++kv)
            for (int64_t t = 0; t < Tnew; ++t) {
                const int64_t row = ((b * Hkv + kv) * Tnew + t) * d;
                const double pos = (double)(start_pos + t);
                for (int64_t i = 0; i < d; ++i) v_out[row + i] = load_elem(v_new, dtype, row + i);
                for (int64_t i = 0; i < h; ++i) {
                    const double x0 = load_elem(k_new, dtype, row + i);
                    const double x1 = load_elem(k_new, dtype, row + i + h);
                    if (base <= 0.0) {
                        k_out[row + i] = x0;
                        k_out[row + i + h] = x1;
                        continue;
                    }
                    const double a = pos * pow(base, -2.0 * (double)i / (double)d);
                    k_out[row + i] = x0 * cos(a) - x1 * sin(a);
                    k_out[row + i + h] = x1 * cos(a) + x0 * sin(a);
                }
            }
    return 0;
}

/* The same without a local window. */
int oracle_attention(const void* q, const void* k, const void* v, int dtype,
                     int64_t B, int64_t H, int64_t Hkv, int64_t Tq, int64_t S,
                     int64_t S_cap, int64_t d, int64_t start_pos, double scale,
                     int causal, const int64_t* rows, int64_t nrows, double* out,
                     double* lse, double* probs, int nthreads) {
    return oracle_attention_window(q, k, v, dtype, B, H, Hkv, Tq, S, S_cap, d, start_pos, scale,
                                   causal, 0, rows, nrows, out, lse, probs, nthreads);
}
