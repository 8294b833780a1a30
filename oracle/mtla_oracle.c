/*
 * mtla_oracle.c -- plain float64 CPU oracle for the MTLA attention hot path.
 *
 * TEST INFRASTRUCTURE. This file is the yardstick the CUDA path is checked
 * against; it is not part of the product. Only the tests, the smoke check in
 * the repository's entry module and the benchmark's CPU-baseline leg load it.
 * It shares no code, header, table or helper with the CUDA library, and it
 * never calls it.
 *
 * What it follows (page titles and the sections they name):
 *   [MTLA]  "Multi-head Temporal Latent Attention" (paper summary page):
 *           Method -- (1) hyper-network merging weights W_t from the latent
 *           times a positional embedding (Sec. 4.1, Eq. 13); in-place update of
 *           the slot still being filled during inference; (2) the stride-aware
 *           causal mask (Sec. 4.2, Fig. 2(c)); (3) decoupled-RoPE keys merged
 *           along the same axis with the same mask (Sec. 4.3, Eq. 17); matrix
 *           absorption of W^UK and W^UV kept from MLA.
 *           Key claims -- the cache holds 9/(4s) elements per token at
 *           d_c = 4 d_h, d_R = d_h/2 (Sec. 4.3).
 *   [MLA]   "Multi-Head Latent Attention and Sparse Indexers", section
 *           "Latent attention changes the representation": the absorption
 *           identities q.(U_K c) = (U_K^T q).c and sum a U_V c = U_V sum a c.
 *
 * Readings taken where the pages are silent or garbled (each is a named
 * choice, not something the pages fix):
 *   - slots are 0-based: token t lives in slot floor(t/s); a sequence of n
 *     tokens owns ceil(n/s) slots;
 *   - query i attends every finished slot j < floor(i/s) plus its own partial
 *     slot P_i = sum_{u = s*floor(i/s)}^{i} w_u x_u (the garbled mask sentence
 *     of Sec. 4.2 read as "finished slots, plus the slot being filled");
 *   - W_t is a linear layer d_c -> s (+ bias) on c_t * PE_t followed by a
 *     sigmoid; token t uses output t mod s as one scalar that scales the whole
 *     vector x_t = [c_t ; RoPE_t(k_t)];
 *   - PE_t is the interleaved sinusoid PE[2k] = sin(t b^(-2k/d_c)),
 *     PE[2k+1] = cos(...), b = 10000, over the latent width d_c;
 *   - RoPE rotates interleaved pairs (x_2k, x_2k+1) by t * base^(-2k/d_R);
 *     keys are rotated at their own position before merging, queries at
 *     theirs;
 *   - scores use scale 1/sqrt(d_h + d_R) unless a scale is given;
 *   - the merged sum is not normalised.
 * Per-channel variant (reading of W_t (.) x_t with W_t a vector): one weight
 * per slot channel, w_t[k] = sigmoid((c_t (.) PE_t) . G[t mod s][:, k] +
 * g[t mod s][k]) with G [s, d_c, D], or the D weights given per token; the
 * scalar modes are the case of equal channels.
 * The PE, RoPE-frequency and gate conventions above are readings (the pages
 * print no worked example of them); the pins hold this file to the exact
 * values those readings give at small sizes (frequencies 1, 0.1, 0.01, 0.001
 * at width 8, a gate value worked by hand), besides their invariants.
 *
 * Everything is float64, written as the definitions read, with no blocking,
 * fusion or reordering. Layouts are row-major:
 *   c [B,T,d_c]  kr [B,T,d_r]  qc [B,T,H,d_h]  qr [B,T,H,d_r]
 *   w_uk, w_uv [H,d_h,d_c]   G [s,d_c]   g [s]   gate_in [B,T]
 *   slot vectors have width D = d_c + d_r: [latent ; rotated key].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_GATE_COMPUTED 0
#define ORC_GATE_SUPPLIED 1
#define ORC_GATE_UNIT 2
#define ORC_GATE_CHANNEL_COMPUTED 3
#define ORC_GATE_CHANNEL_SUPPLIED 4

typedef struct {
    int32_t B, H, d_h, d_c, d_r, s;
    int32_t gate_mode;
    double scale;     /* 0 => 1/sqrt(d_h + d_r) */
    double rope_base; /* base of the decoupled-RoPE frequencies */
    double pe_base;   /* base of the sinusoidal positional embedding */
} orc_cfg;

/* Planted mistakes, used only by the tests that show the pins catch them.
 * 0 means the oracle as written. */
enum {
    ORC_FAULT_NONE = 0,
    ORC_FAULT_DROP_OWN_PARTIAL = 1,  /* forget the slot being filled        */
    ORC_FAULT_MASK_OFF_BY_ONE = 2,   /* let query see finished slot floor(i/s) too */
    ORC_FAULT_TRANSPOSE_WUK = 3,     /* index W^UK as [d_c,d_h]             */
    ORC_FAULT_ROPE_SIGN = 4,         /* rotate the wrong way                */
    ORC_FAULT_SCAN_NO_RESET = 5,     /* never start a fresh slot            */
    ORC_FAULT_DROP_ROPE_KEY = 6,     /* score only the latent part          */
    ORC_FAULT_GATE_WRONG_ROW = 7,    /* use gate row (t+1) mod s            */
    ORC_FAULT_SCALE = 8,             /* scale by 1/sqrt(d_h)                */
    ORC_FAULT_FREQ_EXPONENT = 9,     /* PE and RoPE frequencies base^(-k/d)  */
    ORC_FAULT_PE_BASE = 10,          /* PE with base 1000                    */
    ORC_FAULT_PAIR_ORDER = 11,       /* frequencies of pairs k >= 1 reversed */
    ORC_FAULT_ROPE_HALF_SPLIT = 12,  /* RoPE pairs (x_k, x_{k+d/2})          */
    ORC_FAULT_PE_SWAP = 13,          /* PE with cos at even, sin at odd      */
    ORC_FAULT_CHUNK_NO_SEED = 14,    /* chunked prefill: open block restarts  */
    ORC_FAULT_CHUNK_LOCAL_POS = 15,  /* chunked prefill: positions from 0     */
    ORC_FAULT_CHANNEL_TRANSPOSE = 16, /* per-channel gate read as G [s,D,d_c] */
    ORC_FAULT_BWD_NO_DELTA = 17,     /* backward: softmax gradient without -delta */
    ORC_FAULT_BWD_PREFIX_SUM = 18,   /* backward: scan reversed as prefix sums   */
    ORC_FAULT_BWD_NO_SIGMOID = 19,   /* backward: gate without sigma'            */
};
static int orc_fault = ORC_FAULT_NONE;
void orc_set_fault(int f) { orc_fault = f; }

static double orc_scale(const orc_cfg* cfg) {
    if (orc_fault == ORC_FAULT_SCALE) return 1.0 / sqrt((double)cfg->d_h);
    return cfg->scale != 0.0 ? cfg->scale : 1.0 / sqrt((double)(cfg->d_h + cfg->d_r));
}

/* Inverse frequency base^(-2k/d) of rotation pair k (the reading of the
 * PE and of RoPE), with the planted schedule mistakes of the tests. */
static double orc_inv_freq(int32_t k, int32_t d, double base) {
    if (orc_fault == ORC_FAULT_PAIR_ORDER && k >= 1) k = d / 2 - k;
    double e = (orc_fault == ORC_FAULT_FREQ_EXPONENT) ? -(double)k / d : -2.0 * k / d;
    return pow(base, e);
}

/* Sinusoidal positional embedding of width d at position t. */
void orc_pe(int64_t t, int32_t d, double base, double* pe) {
    if (orc_fault == ORC_FAULT_PE_BASE) base = 1000.0;
    for (int32_t k = 0; 2 * k < d; ++k) {
        double ang = (double)t * orc_inv_freq(k, d, base);
        double even = sin(ang), odd = cos(ang);
        if (orc_fault == ORC_FAULT_PE_SWAP) even = cos(ang), odd = sin(ang);
        pe[2 * k] = even;
        if (2 * k + 1 < d) pe[2 * k + 1] = odd;
    }
}

/* Rotary embedding of a d-vector at position t (interleaved pairs). */
void orc_rope(int64_t t, int32_t d, double base, const double* x, double* y) {
    for (int32_t k = 0; k < d / 2; ++k) {
        double ang = (double)t * orc_inv_freq(k, d, base);
        if (orc_fault == ORC_FAULT_ROPE_SIGN) ang = -ang;
        double cs = cos(ang), sn = sin(ang);
        int32_t i0 = 2 * k, i1 = 2 * k + 1;
        if (orc_fault == ORC_FAULT_ROPE_HALF_SPLIT) i0 = k, i1 = k + d / 2;
        double x0 = x[i0], x1 = x[i1];
        y[i0] = x0 * cs - x1 * sn;
        y[i1] = x0 * sn + x1 * cs;
    }
}

void orc_gate_channels(const orc_cfg* cfg, int64_t t, const double* c_t, const double* G,
                       const double* g, const double* w_given, double* wv);

/* Merging weight of token t (MTLA Sec. 4.1, Eq. 13, under the reading above).
 * w_given points at the supplied weight in SUPPLIED mode. */
double orc_gate(const orc_cfg* cfg, int64_t t, const double* c_t, const double* G,
                const double* g, const double* w_given) {
    if (cfg->gate_mode == ORC_GATE_UNIT) return 1.0;
    if (cfg->gate_mode == ORC_GATE_SUPPLIED) return *w_given;
    if (cfg->gate_mode >= ORC_GATE_CHANNEL_COMPUTED) {
        /* the per-channel modes: the weight of channel 0 (the w outputs below) */
        double* wv = (double*)malloc(sizeof(double) * (cfg->d_c + cfg->d_r));
        orc_gate_channels(cfg, t, c_t, G, g, w_given, wv);
        double w0 = wv[0];
        free(wv);
        return w0;
    }
    int32_t d_c = cfg->d_c;
    int64_t r = t % cfg->s;
    if (orc_fault == ORC_FAULT_GATE_WRONG_ROW) r = (t + 1) % cfg->s;
    double* pe = (double*)malloc(sizeof(double) * d_c);
    orc_pe(t, d_c, cfg->pe_base, pe);
    double z = g[r];
    for (int32_t i = 0; i < d_c; ++i) z += G[r * d_c + i] * (c_t[i] * pe[i]);
    free(pe);
    return 1.0 / (1.0 + exp(-z));
}

/* Per-channel merging weights: the reading of W_t (.) x_t with one weight per
 * slot channel (the latent and the rotated key alike):
 *   w_t[k] = sigmoid( sum_i (c_t (.) PE_t)[i] G[r][i][k] + g[r][k] ),  r = t mod s,
 * G [s, d_c, D], g [s, D] (CHANNEL_COMPUTED), or the D given weights
 * (CHANNEL_SUPPLIED). The scalar modes give their one weight in every channel. */
void orc_gate_channels(const orc_cfg* cfg, int64_t t, const double* c_t, const double* G,
                       const double* g, const double* w_given, double* wv) {
    const int32_t d_c = cfg->d_c, D = cfg->d_c + cfg->d_r;
    if (cfg->gate_mode == ORC_GATE_CHANNEL_SUPPLIED) {
        for (int32_t k = 0; k < D; ++k) wv[k] = w_given[k];
        return;
    }
    if (cfg->gate_mode != ORC_GATE_CHANNEL_COMPUTED) {
        double w = orc_gate(cfg, t, c_t, G, g, w_given);
        for (int32_t k = 0; k < D; ++k) wv[k] = w;
        return;
    }
    int64_t r = t % cfg->s;
    if (orc_fault == ORC_FAULT_GATE_WRONG_ROW) r = (t + 1) % cfg->s;
    double* pe = (double*)malloc(sizeof(double) * d_c);
    orc_pe(t, d_c, cfg->pe_base, pe);
    for (int32_t k = 0; k < D; ++k) {
        double z = g[r * D + k];
        for (int32_t i = 0; i < d_c; ++i) {
            double gik = G[(r * d_c + i) * D + k];
            if (orc_fault == ORC_FAULT_CHANNEL_TRANSPOSE) {
                int64_t flat = (int64_t)i * D + k;          /* read as if stored [D, d_c] */
                gik = G[r * d_c * D + (flat % d_c) * D + flat / d_c];
            }
            z += (c_t[i] * pe[i]) * gik;
        }
        wv[k] = 1.0 / (1.0 + exp(-z));
    }
    free(pe);
}

/* Where the supplied weights of token (b, t) start in gate_in: [B,T] scalars
 * or [B,T,D] per-channel weights. */
static const double* orc_given(const orc_cfg* cfg, const double* gate_in, int64_t bt) {
    if (!gate_in) return NULL;
    return cfg->gate_mode == ORC_GATE_CHANNEL_SUPPLIED ? &gate_in[bt * (cfg->d_c + cfg->d_r)] : &gate_in[bt];
}

/* x_t = [c_t ; RoPE_t(k_t)], the vector a token contributes to its slot. */
static void orc_token_vector(const orc_cfg* cfg, int64_t t, const double* c_t,
                             const double* k_t, double* x) {
    memcpy(x, c_t, sizeof(double) * cfg->d_c);
    orc_rope(t, cfg->d_r, cfg->rope_base, k_t, x + cfg->d_c);
}

/* Block-prefix partial slots (MTLA Sec. 4.2-4.3):
 *   P_t = sum_{u = s*floor(t/s)}^{t} w_u x_u,
 * written out as that sum for every t. Also returns w [B,T]. */
void orc_partials(const orc_cfg* cfg, int32_t T, const double* c, const double* kr,
                  const double* G, const double* g, const double* gate_in,
                  double* w, double* P) {
    const int32_t B = cfg->B, d_c = cfg->d_c, d_r = cfg->d_r, s = cfg->s;
    const int32_t D = d_c + d_r;
    for (int32_t b = 0; b < B; ++b)
        for (int32_t t = 0; t < T; ++t) {
            const int64_t bt = (int64_t)b * T + t;
            w[bt] = orc_gate(cfg, t, &c[bt * d_c], G, g, orc_given(cfg, gate_in, bt));
        }
#pragma omp parallel for schedule(static)
    for (int64_t bt = 0; bt < (int64_t)B * T; ++bt) {
        int32_t b = (int32_t)(bt / T), t = (int32_t)(bt % T);
        double* x = (double*)malloc(sizeof(double) * D);
        double* wv = (double*)malloc(sizeof(double) * D);
        double* out = &P[bt * D];
        for (int32_t k = 0; k < D; ++k) out[k] = 0.0;
        int32_t u0 = s * (t / s);
        if (orc_fault == ORC_FAULT_SCAN_NO_RESET) u0 = 0;
        for (int32_t u = u0; u <= t; ++u) {
            int64_t bu = (int64_t)b * T + u;
            orc_token_vector(cfg, u, &c[bu * d_c], &kr[bu * d_r], x);
            orc_gate_channels(cfg, u, &c[bu * d_c], G, g, orc_given(cfg, gate_in, bu), wv);
            for (int32_t k = 0; k < D; ++k) out[k] += wv[k] * x[k];
        }
        free(wv);
        free(x);
    }
}

/* Absorbed query (MLA absorption, W^UK folded into the query):
 *   qt = [ W_UK[h]^T qC ; RoPE_t(qR) ]   (width D). */
static void orc_absorb_query(const orc_cfg* cfg, int64_t t, int32_t h, const double* qc_h,
                             const double* qr_h, const double* w_uk, double* qt) {
    const int32_t d_h = cfg->d_h, d_c = cfg->d_c;
    const double* W = &w_uk[(int64_t)h * d_h * d_c];
    for (int32_t j = 0; j < d_c; ++j) {
        double acc = 0.0;
        for (int32_t i = 0; i < d_h; ++i) {
            double wij = W[(int64_t)i * d_c + j];
            if (orc_fault == ORC_FAULT_TRANSPOSE_WUK) {
                int64_t flat = (int64_t)i * d_c + j; /* read as if stored [d_c, d_h] */
                wij = W[(flat % d_h) * d_c + flat / d_h];
            }
            acc += wij * qc_h[i];
        }
        qt[j] = acc;
    }
    orc_rope(t, cfg->d_r, cfg->rope_base, qr_h, qt + d_c);
}

/* Softmax attention of one absorbed query over n key vectors (width D);
 * returns o_lat = sum_k a_k key_k[0:d_c]. */
static void orc_attend_keys(const orc_cfg* cfg, const double* qt, int64_t n,
                            const double* const* keys, double* olat) {
    const int32_t d_c = cfg->d_c, D = cfg->d_c + cfg->d_r;
    const double scale = orc_scale(cfg);
    double* e = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double m = -INFINITY;
    int32_t score_width = (orc_fault == ORC_FAULT_DROP_ROPE_KEY) ? d_c : D;
    for (int64_t k = 0; k < n; ++k) {
        double acc = 0.0;
        for (int32_t j = 0; j < score_width; ++j) acc += qt[j] * keys[k][j];
        e[k] = scale * acc;
        if (e[k] > m) m = e[k];
    }
    double l = 0.0;
    for (int64_t k = 0; k < n; ++k) {
        e[k] = exp(e[k] - m);
        l += e[k];
    }
    for (int32_t j = 0; j < d_c; ++j) olat[j] = 0.0;
    for (int64_t k = 0; k < n; ++k)
        for (int32_t j = 0; j < d_c; ++j) olat[j] += (e[k] / l) * keys[k][j];
    free(e);
}

/* Output absorption: o = W_UV[h] o_lat (width d_h). */
static void orc_output(const orc_cfg* cfg, int32_t h, const double* olat, const double* w_uv,
                       double* o) {
    const int32_t d_h = cfg->d_h, d_c = cfg->d_c;
    const double* W = &w_uv[(int64_t)h * d_h * d_c];
    for (int32_t i = 0; i < d_h; ++i) {
        double acc = 0.0;
        for (int32_t j = 0; j < d_c; ++j) acc += W[(int64_t)i * d_c + j] * olat[j];
        o[i] = acc;
    }
}

/* The allowed key set of query i (stride-aware causal mask, MTLA Sec. 4.2):
 * finished slots F_j = P_{js+s-1} for j < floor(i/s), then the own partial
 * P_i. Fills `keys` (room for floor(i/s)+2 pointers); returns the count. */
static int64_t orc_allowed_keys(const orc_cfg* cfg, int32_t T, const double* P_b, int32_t i,
                                const double** keys) {
    const int32_t s = cfg->s, D = cfg->d_c + cfg->d_r;
    int64_t n = 0;
    int32_t nf = i / s;
    if (orc_fault == ORC_FAULT_MASK_OFF_BY_ONE) nf = i / s + 1;
    for (int32_t j = 0; j < nf; ++j) {
        int32_t u = j * s + s - 1;
        if (u >= T) u = T - 1;
        keys[n++] = &P_b[(int64_t)u * D];
    }
    if (orc_fault != ORC_FAULT_DROP_OWN_PARTIAL) keys[n++] = &P_b[(int64_t)i * D];
    return n;
}

/* Parallel (training-form) attention for selected rows (b, t), all heads.
 * P is the output of orc_partials. rows holds n_rows pairs (b, t).
 * out [n_rows,H,d_h]; olat [n_rows,H,d_c] may be NULL. */
void orc_attend_rows(const orc_cfg* cfg, int32_t T, const double* qc, const double* qr,
                     const double* w_uk, const double* w_uv, const double* P, int64_t n_rows,
                     const int64_t* rows, double* out, double* olat_out) {
    const int32_t H = cfg->H, d_h = cfg->d_h, d_c = cfg->d_c, d_r = cfg->d_r;
    const int32_t D = d_c + d_r;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t rh = 0; rh < n_rows * H; ++rh) {
        int64_t r = rh / H;
        int32_t h = (int32_t)(rh % H);
        int32_t b = (int32_t)rows[2 * r], t = (int32_t)rows[2 * r + 1];
        int64_t bth = ((int64_t)b * T + t) * H + h;
        double* qt = (double*)malloc(sizeof(double) * D);
        double* olat = (double*)malloc(sizeof(double) * d_c);
        const double** keys = (const double**)malloc(sizeof(double*) * (size_t)(t / cfg->s + 2));
        orc_absorb_query(cfg, t, h, &qc[bth * d_h], &qr[bth * d_r], w_uk, qt);
        int64_t n = orc_allowed_keys(cfg, T, &P[(int64_t)b * T * D], t, keys);
        orc_attend_keys(cfg, qt, n, keys, olat);
        orc_output(cfg, h, olat, w_uv, &out[(r * H + h) * d_h]);
        if (olat_out) memcpy(&olat_out[(r * H + h) * d_c], olat, sizeof(double) * d_c);
        free(keys);
        free(olat);
        free(qt);
    }
}

/* Full parallel forward over T tokens from position 0.
 * out [B,T,H,d_h]; w [B,T]; cache [B,ceil(T/s),D] = the cache after T tokens
 * (finished slots, then the last, possibly partial, slot); acc [B,D] = P_{T-1}. */
void orc_prefill(const orc_cfg* cfg, int32_t T, const double* c, const double* kr,
                 const double* qc, const double* qr, const double* w_uk, const double* w_uv,
                 const double* G, const double* g, const double* gate_in, double* out,
                 double* w, double* cache, double* acc) {
    const int32_t B = cfg->B, s = cfg->s, D = cfg->d_c + cfg->d_r;
    const int32_t n_slots = (T + s - 1) / s;
    double* P = (double*)malloc(sizeof(double) * (size_t)B * T * D);
    orc_partials(cfg, T, c, kr, G, g, gate_in, w, P);
    int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * 2 * (size_t)B * T);
    for (int32_t b = 0; b < B; ++b)
        for (int32_t t = 0; t < T; ++t) {
            rows[2 * ((int64_t)b * T + t)] = b;
            rows[2 * ((int64_t)b * T + t) + 1] = t;
        }
    orc_attend_rows(cfg, T, qc, qr, w_uk, w_uv, P, (int64_t)B * T, rows, out, NULL);
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t j = 0; j < n_slots; ++j) {
            int32_t u = j * s + s - 1;
            if (u > T - 1) u = T - 1;
            memcpy(&cache[((int64_t)b * n_slots + j) * D], &P[((int64_t)b * T + u) * D],
                   sizeof(double) * D);
        }
        if (T > 0)
            memcpy(&acc[(int64_t)b * D], &P[((int64_t)b * T + T - 1) * D], sizeof(double) * D);
    }
    free(rows);
    free(P);
}

/* Parallel forward over T new tokens at positions t0 .. t0+T-1 that continues
 * from the state after t0 tokens (chunked prefill): the finished slots
 * F_0 .. F_{floor(t0/s)-1} are cache_in's, and the block open at t0 (when t0 is
 * not a multiple of s) continues from acc_in = P_{t0-1}:
 *   P_i = [s*floor(i/s) < t0 ? acc_in : 0] + sum_{u = max(t0, s*floor(i/s))}^{i} w_u x_u.
 * Query i attends F_j, j < floor(i/s) (cache_in's for j < floor(t0/s), the new
 * block ends otherwise), plus P_i -- the same mask and the same sums as the
 * parallel form over all t0+T tokens (MTLA Sec. 4.2).
 *   cache_in [B,n_in,D] (n_in >= floor(t0/s))   acc_in [B,D]
 *   c [B,T,d_c] kr [B,T,d_r] qc [B,T,H,d_h] qr [B,T,H,d_r] gate_in [B,T]: the new tokens
 *   out [B,T,H,d_h]; w [B,T]; cache_out [B,ceil((t0+T)/s),D] = the cache after
 *   t0+T tokens (cache_in's finished slots, then the new ones); acc_out [B,D]. */
void orc_prefill_from(const orc_cfg* cfg, int32_t t0, int32_t T, int32_t n_in, const double* cache_in,
                      const double* acc_in, const double* c, const double* kr, const double* qc,
                      const double* qr, const double* w_uk, const double* w_uv, const double* G,
                      const double* g, const double* gate_in, double* out, double* w, double* cache_out,
                      double* acc_out) {
    const int32_t B = cfg->B, H = cfg->H, d_h = cfg->d_h, d_c = cfg->d_c, d_r = cfg->d_r, s = cfg->s;
    const int32_t D = d_c + d_r;
    const int32_t nf0 = t0 / s;                         /* finished slots before the chunk */
    const int32_t n_out = (t0 + T + s - 1) / s;
    double* P = (double*)malloc(sizeof(double) * (size_t)B * T * D);
    /* gates, then the partial slots of the new positions (local index i - t0) */
    for (int32_t b = 0; b < B; ++b)
        for (int32_t li = 0; li < T; ++li) {
            const int64_t bl = (int64_t)b * T + li;
            w[bl] = orc_gate(cfg, t0 + li, &c[bl * d_c], G, g, orc_given(cfg, gate_in, bl));
        }
#pragma omp parallel for schedule(static)
    for (int64_t bl = 0; bl < (int64_t)B * T; ++bl) {
        const int32_t b = (int32_t)(bl / T), li = (int32_t)(bl % T), i = t0 + li;
        double* x = (double*)malloc(sizeof(double) * D);
        double* wv = (double*)malloc(sizeof(double) * D);
        double* o = &P[bl * D];
        int32_t u0 = s * (i / s);
        if (orc_fault == ORC_FAULT_SCAN_NO_RESET) u0 = 0;
        const int seeded = u0 < t0 && orc_fault != ORC_FAULT_CHUNK_NO_SEED;
        for (int32_t k = 0; k < D; ++k) o[k] = seeded ? acc_in[(int64_t)b * D + k] : 0.0;
        for (int32_t u = u0 < t0 ? t0 : u0; u <= i; ++u) {
            const int64_t bu = (int64_t)b * T + (u - t0);
            const int32_t tu = orc_fault == ORC_FAULT_CHUNK_LOCAL_POS ? u - t0 : u;
            orc_token_vector(cfg, tu, &c[bu * d_c], &kr[bu * d_r], x);
            orc_gate_channels(cfg, tu, &c[bu * d_c], G, g, orc_given(cfg, gate_in, bu), wv);
            for (int32_t k = 0; k < D; ++k) o[k] += wv[k] * x[k];
        }
        free(wv);
        free(x);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t blh = 0; blh < (int64_t)B * T * H; ++blh) {
        const int32_t h = (int32_t)(blh % H), li = (int32_t)((blh / H) % T), b = (int32_t)(blh / ((int64_t)H * T));
        const int32_t i = t0 + li;
        double* qt = (double*)malloc(sizeof(double) * D);
        double* olat = (double*)malloc(sizeof(double) * d_c);
        const double** keys = (const double**)malloc(sizeof(double*) * (size_t)(i / s + 2));
        int64_t n = 0;
        int32_t nf = i / s;
        if (orc_fault == ORC_FAULT_MASK_OFF_BY_ONE) nf = i / s + 1;
        for (int32_t j = 0; j < nf; ++j) {
            if (j < nf0) {
                keys[n++] = &cache_in[((int64_t)b * n_in + j) * D];
            } else {
                int32_t u = j * s + s - 1;
                if (u > t0 + T - 1) u = t0 + T - 1;
                keys[n++] = &P[((int64_t)b * T + (u - t0)) * D];
            }
        }
        if (orc_fault != ORC_FAULT_DROP_OWN_PARTIAL) keys[n++] = &P[((int64_t)b * T + li) * D];
        orc_absorb_query(cfg, i, h, &qc[blh * d_h], &qr[blh * d_r], w_uk, qt);
        orc_attend_keys(cfg, qt, n, keys, olat);
        orc_output(cfg, h, olat, w_uv, &out[blh * d_h]);
        free(keys);
        free(olat);
        free(qt);
    }
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t j = 0; j < n_out; ++j) {
            double* dst = &cache_out[((int64_t)b * n_out + j) * D];
            if (j < nf0) {
                memcpy(dst, &cache_in[((int64_t)b * n_in + j) * D], sizeof(double) * D);
            } else {
                int32_t u = j * s + s - 1;
                if (u > t0 + T - 1) u = t0 + T - 1;
                memcpy(dst, &P[((int64_t)b * T + (u - t0)) * D], sizeof(double) * D);
            }
        }
        memcpy(&acc_out[(int64_t)b * D], &P[((int64_t)b * T + T - 1) * D], sizeof(double) * D);
    }
    free(P);
}

/* One incremental decode step (MTLA Sec. 4.1 inference): token t = pos[b]
 * of every sequence. Opens a fresh slot when t mod s == 0, otherwise adds
 * into the slot being filled in place; then the query attends slots
 * 0..floor(t/s) of the cache.
 *   c_new [B,d_c]  kr_new [B,d_r]  qc [B,H,d_h]  qr [B,H,d_r]  gate_in [B]
 *   cache [B,max_slots,D] in/out   acc [B,D] in/out   out [B,H,d_h]
 *   w_out [B] and olat_out [B,H,d_c] may be NULL. */
void orc_decode_step(const orc_cfg* cfg, int32_t max_slots, const double* c_new,
                     const double* kr_new, const double* qc, const double* qr,
                     const double* w_uk, const double* w_uv, const double* G, const double* g,
                     const double* gate_in, const int64_t* pos, double* cache, double* acc,
                     double* out, double* w_out, double* olat_out) {
    const int32_t B = cfg->B, H = cfg->H, d_h = cfg->d_h, d_c = cfg->d_c, d_r = cfg->d_r;
    const int32_t s = cfg->s, D = d_c + d_r;
    for (int32_t b = 0; b < B; ++b) {
        int64_t t = pos[b];
        int64_t j = t / s;
        const double* wg = orc_given(cfg, gate_in, b);
        double* wv = (double*)malloc(sizeof(double) * D);
        orc_gate_channels(cfg, t, &c_new[(int64_t)b * d_c], G, g, wg, wv);
        if (w_out) w_out[b] = wv[0];
        double* x = (double*)malloc(sizeof(double) * D);
        orc_token_vector(cfg, t, &c_new[(int64_t)b * d_c], &kr_new[(int64_t)b * d_r], x);
        double* a = &acc[(int64_t)b * D];
        int fresh = (t % s == 0);
        if (orc_fault == ORC_FAULT_SCAN_NO_RESET) fresh = (t == 0);
        for (int32_t k = 0; k < D; ++k) a[k] = (fresh ? 0.0 : a[k]) + wv[k] * x[k];
        memcpy(&cache[((int64_t)b * max_slots + j) * D], a, sizeof(double) * D);
        free(x);
        free(wv);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        int32_t b = (int32_t)(bh / H), h = (int32_t)(bh % H);
        int64_t t = pos[b];
        int64_t n = t / s + 1;
        if (orc_fault == ORC_FAULT_DROP_OWN_PARTIAL) n = t / s;
        double* qt = (double*)malloc(sizeof(double) * D);
        double* olat = (double*)malloc(sizeof(double) * d_c);
        const double** keys = (const double**)malloc(sizeof(double*) * (size_t)(n > 0 ? n : 1));
        for (int64_t k = 0; k < n; ++k) keys[k] = &cache[((int64_t)b * max_slots + k) * D];
        orc_absorb_query(cfg, t, h, &qc[bh * d_h], &qr[bh * d_r], w_uk, qt);
        orc_attend_keys(cfg, qt, n, keys, olat);
        orc_output(cfg, h, olat, w_uv, &out[bh * d_h]);
        if (olat_out) memcpy(&olat_out[bh * d_c], olat, sizeof(double) * d_c);
        free(keys);
        free(olat);
        free(qt);
    }
}

/* The same parallel forward written without absorption: every allowed slot
 * is expanded to an explicit per-head key k = [W_UK[h] F[0:d_c] ; F[d_c:]]
 * and value v = W_UV[h] F[0:d_c]; the query is [qC ; RoPE_t(qR)]. Used to
 * check the absorbed form (MLA absorption identities). out [B,T,H,d_h]. */
void orc_prefill_explicit(const orc_cfg* cfg, int32_t T, const double* c, const double* kr,
                          const double* qc, const double* qr, const double* w_uk,
                          const double* w_uv, const double* G, const double* g,
                          const double* gate_in, double* out) {
    const int32_t B = cfg->B, H = cfg->H, d_h = cfg->d_h, d_c = cfg->d_c, d_r = cfg->d_r;
    const int32_t D = d_c + d_r;
    const double scale = orc_scale(cfg);
    double* P = (double*)malloc(sizeof(double) * (size_t)B * T * D);
    double* w = (double*)malloc(sizeof(double) * (size_t)B * T);
    orc_partials(cfg, T, c, kr, G, g, gate_in, w, P);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bth = 0; bth < (int64_t)B * T * H; ++bth) {
        int32_t h = (int32_t)(bth % H);
        int32_t t = (int32_t)((bth / H) % T);
        int32_t b = (int32_t)(bth / ((int64_t)H * T));
        const double* Wk = &w_uk[(int64_t)h * d_h * d_c];
        const double* Wv = &w_uv[(int64_t)h * d_h * d_c];
        double* q = (double*)malloc(sizeof(double) * (d_h + d_r));
        memcpy(q, &qc[bth * d_h], sizeof(double) * d_h);
        orc_rope(t, d_r, cfg->rope_base, &qr[bth * d_r], q + d_h);
        const double** keys = (const double**)malloc(sizeof(double*) * (size_t)(t / cfg->s + 2));
        int64_t n = orc_allowed_keys(cfg, T, &P[(int64_t)b * T * D], t, keys);
        double* e = (double*)malloc(sizeof(double) * (size_t)n);
        double* kfull = (double*)malloc(sizeof(double) * (d_h + d_r));
        double m = -INFINITY;
        for (int64_t k = 0; k < n; ++k) {
            for (int32_t i = 0; i < d_h; ++i) {
                double acc = 0.0;
                for (int32_t j = 0; j < d_c; ++j) acc += Wk[(int64_t)i * d_c + j] * keys[k][j];
                kfull[i] = acc;
            }
            for (int32_t r = 0; r < d_r; ++r) kfull[d_h + r] = keys[k][d_c + r];
            double dot = 0.0;
            for (int32_t i = 0; i < d_h + d_r; ++i) dot += q[i] * kfull[i];
            e[k] = scale * dot;
            if (e[k] > m) m = e[k];
        }
        double l = 0.0;
        for (int64_t k = 0; k < n; ++k) {
            e[k] = exp(e[k] - m);
            l += e[k];
        }
        double* o = &out[bth * d_h];
        for (int32_t i = 0; i < d_h; ++i) o[i] = 0.0;
        for (int64_t k = 0; k < n; ++k)
            for (int32_t i = 0; i < d_h; ++i) {
                double v = 0.0;
                for (int32_t j = 0; j < d_c; ++j) v += Wv[(int64_t)i * d_c + j] * keys[k][j];
                o[i] += (e[k] / l) * v;
            }
        free(kfull);
        free(e);
        free(keys);
        free(q);
    }
    free(w);
    free(P);
}

/* Gradients of the parallel forward from position 0 (training), for the
 * scalar gate modes. With o_{i,h} = W_UV[h] obar_{i,h}, obar = sum_j a_ij key_j[0:d_c],
 * a = softmax_j(e), e_ij = scale qt_{i,h} . key_j over the allowed keys of i
 * (finished slots F_j = P_{js+s-1}, j < floor(i/s), and the own partial P_i),
 * qt = [W_UK[h]^T qC ; R_i qR] and P_t = sum_{u in block(t), u <= t} w_u x_u,
 * x_u = [c_u ; R_u k_u], the chain rule taken step by step from dout:
 *   dW_UV[h] += dout obar^T;  dobar = W_UV[h]^T dout;  delta = dobar . obar
 *   de_ij = a_ij (dobar . key_j[0:d_c] - delta)
 *   dqt = scale sum_j de_ij key_j;  dkey_j += scale de_ij qt + a_ij [dobar ; 0]
 *   dqC = W_UK[h] dqt[0:d_c];  dW_UK[h] += qC dqt[0:d_c]^T;  dqR = R_i^T dqt[d_c:]
 *   dP_t = (key gradient of P_t as an own partial) + (as F_j when t = js+s-1)
 *   S_u = sum_{t >= u, t in block(u)} dP_t;  dx_u = w_u S_u;  dw_u = x_u . S_u
 *   dc_u = dx_u[0:d_c];  dk_u = R_u^T dx_u[d_c:]
 *   COMPUTED: dz = dw w (1 - w); dG[r] += dz (c*PE); dg[r] += dz; dc += dz G[r]*PE
 *   SUPPLIED: dgate_in = dw.
 * Outputs (zeroed here): dc [B,T,d_c] dkr [B,T,d_r] dqc [B,T,H,d_h] dqr [B,T,H,d_r]
 * dw_uk, dw_uv [H,d_h,d_c] dG [s,d_c] dg [s] dgate_in [B,T] (NULL where unused). */
void orc_prefill_backward(const orc_cfg* cfg, int32_t T, const double* c, const double* kr, const double* qc,
                          const double* qr, const double* w_uk, const double* w_uv, const double* G,
                          const double* g, const double* gate_in, const double* dout, double* dc, double* dkr,
                          double* dqc, double* dqr, double* dw_uk, double* dw_uv, double* dG, double* dg,
                          double* dgate_in) {
    const int32_t B = cfg->B, H = cfg->H, d_h = cfg->d_h, d_c = cfg->d_c, d_r = cfg->d_r, s = cfg->s;
    const int32_t D = d_c + d_r;
    const double scale = orc_scale(cfg);
    double* w = (double*)malloc(sizeof(double) * (size_t)B * T);
    double* P = (double*)malloc(sizeof(double) * (size_t)B * T * D);
    double* dP = (double*)calloc((size_t)B * T * D, sizeof(double));
    orc_partials(cfg, T, c, kr, G, g, gate_in, w, P);
    memset(dc, 0, sizeof(double) * (size_t)B * T * d_c);
    memset(dkr, 0, sizeof(double) * (size_t)B * T * d_r);
    memset(dqc, 0, sizeof(double) * (size_t)B * T * H * d_h);
    memset(dqr, 0, sizeof(double) * (size_t)B * T * H * d_r);
    memset(dw_uk, 0, sizeof(double) * (size_t)H * d_h * d_c);
    memset(dw_uv, 0, sizeof(double) * (size_t)H * d_h * d_c);
    if (dG) memset(dG, 0, sizeof(double) * (size_t)s * d_c);
    if (dg) memset(dg, 0, sizeof(double) * (size_t)s);
    if (dgate_in) memset(dgate_in, 0, sizeof(double) * (size_t)B * T);
    double* qt = (double*)malloc(sizeof(double) * D);
    double* dqt = (double*)malloc(sizeof(double) * D);
    double* obar = (double*)malloc(sizeof(double) * d_c);
    double* dob = (double*)malloc(sizeof(double) * d_c);
    double* e = (double*)malloc(sizeof(double) * (size_t)(T / s + 2));
    int64_t* kidx = (int64_t*)malloc(sizeof(int64_t) * (size_t)(T / s + 2));   /* key -> row of P */
    /* attention, one (b, i, h) at a time (plain loops, no reordering) */
    for (int32_t b = 0; b < B; ++b)
        for (int32_t i = 0; i < T; ++i)
            for (int32_t h = 0; h < H; ++h) {
                const int64_t bih = ((int64_t)b * T + i) * H + h;
                orc_absorb_query(cfg, i, h, &qc[bih * d_h], &qr[bih * d_r], w_uk, qt);
                int64_t n = 0;
                for (int32_t j = 0; j < i / s; ++j) kidx[n++] = (int64_t)b * T + j * s + s - 1;
                if (orc_fault != ORC_FAULT_DROP_OWN_PARTIAL) kidx[n++] = (int64_t)b * T + i;
                double m = -INFINITY;
                for (int64_t k = 0; k < n; ++k) {
                    const double* key = &P[kidx[k] * D];
                    double acc = 0.0;
                    for (int32_t q = 0; q < D; ++q) acc += qt[q] * key[q];
                    e[k] = scale * acc;
                    if (e[k] > m) m = e[k];
                }
                double l = 0.0;
                for (int64_t k = 0; k < n; ++k) {
                    e[k] = exp(e[k] - m);
                    l += e[k];
                }
                for (int64_t k = 0; k < n; ++k) e[k] /= l;               /* a_ij */
                for (int32_t q = 0; q < d_c; ++q) obar[q] = 0.0;
                for (int64_t k = 0; k < n; ++k)
                    for (int32_t q = 0; q < d_c; ++q) obar[q] += e[k] * P[kidx[k] * D + q];
                const double* W_uv = &w_uv[(int64_t)h * d_h * d_c];
                const double* dO = &dout[bih * d_h];
                for (int32_t q = 0; q < d_c; ++q) {
                    double acc = 0.0;
                    for (int32_t r = 0; r < d_h; ++r) acc += W_uv[(int64_t)r * d_c + q] * dO[r];
                    dob[q] = acc;
                }
                for (int32_t r = 0; r < d_h; ++r)
                    for (int32_t q = 0; q < d_c; ++q) dw_uv[((int64_t)h * d_h + r) * d_c + q] += dO[r] * obar[q];
                double delta = 0.0;
                for (int32_t q = 0; q < d_c; ++q) delta += dob[q] * obar[q];
                for (int32_t q = 0; q < D; ++q) dqt[q] = 0.0;
                for (int64_t k = 0; k < n; ++k) {
                    double* key = &P[kidx[k] * D];
                    double* dkey = &dP[kidx[k] * D];
                    double da = 0.0;
                    for (int32_t q = 0; q < d_c; ++q) da += dob[q] * key[q];
                    const double de = e[k] * (da - (orc_fault == ORC_FAULT_BWD_NO_DELTA ? 0.0 : delta));
                    for (int32_t q = 0; q < D; ++q) {
                        dqt[q] += scale * de * key[q];
                        dkey[q] += scale * de * qt[q];
                    }
                    for (int32_t q = 0; q < d_c; ++q) dkey[q] += e[k] * dob[q];
                }
                /* back through the query absorption and the query RoPE */
                const double* W_uk = &w_uk[(int64_t)h * d_h * d_c];
                for (int32_t r = 0; r < d_h; ++r) {
                    double acc = 0.0;
                    for (int32_t q = 0; q < d_c; ++q) {
                        acc += W_uk[(int64_t)r * d_c + q] * dqt[q];
                        dw_uk[((int64_t)h * d_h + r) * d_c + q] += qc[bih * d_h + r] * dqt[q];
                    }
                    dqc[bih * d_h + r] = acc;
                }
                orc_rope(-(int64_t)i, d_r, cfg->rope_base, &dqt[d_c], &dqr[bih * d_r]);   /* R_i^T = R_{-i} */
            }
    /* back through the block-prefix scan and the merging gate */
    double* x = (double*)malloc(sizeof(double) * D);
    double* S = (double*)malloc(sizeof(double) * D);
    double* dx = (double*)malloc(sizeof(double) * D);
    double* pe = (double*)malloc(sizeof(double) * d_c);
    for (int32_t b = 0; b < B; ++b)
        for (int32_t u = 0; u < T; ++u) {
            const int64_t bu = (int64_t)b * T + u;
            const int32_t blk_end = s * (u / s) + s - 1 < T - 1 ? s * (u / s) + s - 1 : T - 1;
            for (int32_t q = 0; q < D; ++q) S[q] = 0.0;
            const int32_t blk0 = s * (u / s);
            for (int32_t t = (orc_fault == ORC_FAULT_BWD_PREFIX_SUM ? blk0 : u);
                 t <= (orc_fault == ORC_FAULT_BWD_PREFIX_SUM ? u : blk_end); ++t)
                for (int32_t q = 0; q < D; ++q) S[q] += dP[((int64_t)b * T + t) * D + q];
            orc_token_vector(cfg, u, &c[bu * d_c], &kr[bu * d_r], x);
            double dw = 0.0;
            for (int32_t q = 0; q < D; ++q) {
                dx[q] = w[bu] * S[q];
                dw += x[q] * S[q];
            }
            for (int32_t q = 0; q < d_c; ++q) dc[bu * d_c + q] += dx[q];
            orc_rope(-(int64_t)u, d_r, cfg->rope_base, &dx[d_c], &dkr[bu * d_r]);
            if (cfg->gate_mode == ORC_GATE_SUPPLIED && dgate_in) dgate_in[bu] = dw;
            if (cfg->gate_mode == ORC_GATE_COMPUTED) {
                const int32_t r = u % s;
                const double dz = orc_fault == ORC_FAULT_BWD_NO_SIGMOID ? dw : dw * w[bu] * (1.0 - w[bu]);
                orc_pe(u, d_c, cfg->pe_base, pe);
                for (int32_t q = 0; q < d_c; ++q) {
                    dG[(int64_t)r * d_c + q] += dz * c[bu * d_c + q] * pe[q];
                    dc[bu * d_c + q] += dz * G[(int64_t)r * d_c + q] * pe[q];
                }
                dg[r] += dz;
            }
        }
    free(pe); free(dx); free(S); free(x); free(kidx); free(e); free(dob); free(obar); free(dqt); free(qt);
    free(dP); free(P); free(w);
}

/* The query-side gradients of selected rows of the same backward: for row
 * (b, i) = (rows_b[r], rows_i[r]), dqc_out[r][h][:] and dqr_out[r][h][:] are
 * the gradients of L = sum(dout * out) with respect to qC[b,i,h,:] and
 * qR[b,i,h,:]. They depend only on that row's query, its keys (the finished
 * slots before it and its own partial) and dout[b,i], so each is computed
 * alone: the row's share of orc_prefill_backward's dqc / dqr, the same steps
 * in the same order (for checks at sizes where the whole backward is too
 * slow). */
void orc_backward_rows(const orc_cfg* cfg, int32_t T, const double* c, const double* kr, const double* qc,
                       const double* qr, const double* w_uk, const double* w_uv, const double* G, const double* g,
                       const double* gate_in, const double* dout, int32_t n_rows, const int32_t* rows_b,
                       const int32_t* rows_i, double* dqc_out, double* dqr_out) {
    const int32_t B = cfg->B, H = cfg->H, d_h = cfg->d_h, d_c = cfg->d_c, d_r = cfg->d_r, s = cfg->s;
    const int32_t D = d_c + d_r;
    const double scale = orc_scale(cfg);
    double* w = (double*)malloc(sizeof(double) * (size_t)B * T);
    double* P = (double*)malloc(sizeof(double) * (size_t)B * T * D);
    orc_partials(cfg, T, c, kr, G, g, gate_in, w, P);
#pragma omp parallel for schedule(dynamic)
    for (int32_t r = 0; r < n_rows; ++r) {
        const int32_t b = rows_b[r], i = rows_i[r];
        double* qt = (double*)malloc(sizeof(double) * D);
        double* dqt = (double*)malloc(sizeof(double) * D);
        double* obar = (double*)malloc(sizeof(double) * d_c);
        double* dob = (double*)malloc(sizeof(double) * d_c);
        double* e = (double*)malloc(sizeof(double) * (size_t)(i / s + 2));
        int64_t* kidx = (int64_t*)malloc(sizeof(int64_t) * (size_t)(i / s + 2));
        for (int32_t h = 0; h < H; ++h) {
            const int64_t bih = ((int64_t)b * T + i) * H + h;
            orc_absorb_query(cfg, i, h, &qc[bih * d_h], &qr[bih * d_r], w_uk, qt);
            int64_t n = 0;
            for (int32_t j = 0; j < i / s; ++j) kidx[n++] = (int64_t)b * T + j * s + s - 1;
            kidx[n++] = (int64_t)b * T + i;
            double m = -INFINITY;
            for (int64_t k = 0; k < n; ++k) {
                double acc = 0.0;
                for (int32_t q = 0; q < D; ++q) acc += qt[q] * P[kidx[k] * D + q];
                e[k] = scale * acc;
                if (e[k] > m) m = e[k];
            }
            double l = 0.0;
            for (int64_t k = 0; k < n; ++k) {
                e[k] = exp(e[k] - m);
                l += e[k];
            }
            for (int64_t k = 0; k < n; ++k) e[k] /= l;
            for (int32_t q = 0; q < d_c; ++q) obar[q] = 0.0;
            for (int64_t k = 0; k < n; ++k)
                for (int32_t q = 0; q < d_c; ++q) obar[q] += e[k] * P[kidx[k] * D + q];
            const double* W_uv = &w_uv[(int64_t)h * d_h * d_c];
            const double* dO = &dout[bih * d_h];
            for (int32_t q = 0; q < d_c; ++q) {
                double acc = 0.0;
                for (int32_t rr = 0; rr < d_h; ++rr) acc += W_uv[(int64_t)rr * d_c + q] * dO[rr];
                dob[q] = acc;
            }
            double delta = 0.0;
            for (int32_t q = 0; q < d_c; ++q) delta += dob[q] * obar[q];
            for (int32_t q = 0; q < D; ++q) dqt[q] = 0.0;
            for (int64_t k = 0; k < n; ++k) {
                const double* key = &P[kidx[k] * D];
                double da = 0.0;
                for (int32_t q = 0; q < d_c; ++q) da += dob[q] * key[q];
                const double de = e[k] * (da - (orc_fault == ORC_FAULT_BWD_NO_DELTA ? 0.0 : delta));
                for (int32_t q = 0; q < D; ++q) dqt[q] += scale * de * key[q];
            }
            const double* W_uk = &w_uk[(int64_t)h * d_h * d_c];
            double* dqc_r = &dqc_out[((int64_t)r * H + h) * d_h];
            for (int32_t rr = 0; rr < d_h; ++rr) {
                double acc = 0.0;
                for (int32_t q = 0; q < d_c; ++q) acc += W_uk[(int64_t)rr * d_c + q] * dqt[q];
                dqc_r[rr] = acc;
            }
            orc_rope(-(int64_t)i, d_r, cfg->rope_base, &dqt[d_c], &dqr_out[((int64_t)r * H + h) * d_r]);
        }
        free(kidx); free(e); free(dob); free(obar); free(dqt); free(qt);
    }
    free(P); free(w);
}

/* y[M, N] = x[M, K] . w[N, K]^T, the definition as three loops (float64). */
void orc_linear(int64_t M, int64_t N, int64_t K, const double* x, const double* w, double* y) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += x[i * K + k] * w[n * K + k];
            y[i * N + n] = acc;
        }
}

/* Beam-search reorder of the cache (the authors' toolkit decodes with
 * parallel beam search: its project page on sourcepulse.org, "Highlighted
 * Details"). Destination b takes over the cache of its parent j = src[b]:
 * the ceil(n_tokens[j] / s) slots j has filled (slot count of n tokens, as
 * above) and j's open-slot accumulator, both copied byte for byte (values of
 * `elem_bytes` bytes in the cache, float32 in the open slot); the other slots
 * of the destination keep their contents. A parent outside [0, B) leaves the
 * destination unchanged and gives status 1, a parent with more tokens than
 * the cache holds gives 3 (the first in b order is returned, 0 if none). */
int orc_reorder_cache(int32_t B, int32_t max_slots, int32_t D, int32_t s, int32_t elem_bytes,
                      const int32_t* src, const int32_t* n_tokens, const unsigned char* cache_in,
                      const float* open_in, unsigned char* cache_out, float* open_out) {
    int status = 0;
    const size_t row_bytes = (size_t)D * (size_t)elem_bytes;
    for (int32_t b = 0; b < B; ++b) {
        const int32_t j = src[b];
        if (j < 0 || j >= B) {
            if (!status) status = 1;
            continue;
        }
        const int64_t n = n_tokens[j];
        if (n < 0 || n > (int64_t)max_slots * s) {
            if (!status) status = 3;
            continue;
        }
        const int64_t slots = (n + s - 1) / s;
        for (int64_t k = 0; k < slots; ++k)
            memcpy(cache_out + ((size_t)b * max_slots + (size_t)k) * row_bytes,
                   cache_in + ((size_t)j * max_slots + (size_t)k) * row_bytes, row_bytes);
        for (int32_t e = 0; e < D; ++e) open_out[(size_t)b * D + e] = open_in[(size_t)j * D + e];
    }
    return status;
}
