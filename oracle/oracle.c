/*
 * oracle.c -- plain CPU reference of the expert-routed (MoE) quantized matmul.
 *
 * TEST INFRASTRUCTURE ONLY. Tests, the package smoke check and the benchmark's
 * CPU-baseline / reference legs load this library; the product path (the CUDA
 * library and its Python binding) never loads, calls or links it, and shares no
 * code, header or table with it.
 *
 * What it computes (mlx-native 0.1.0, src/ops/quantized_matmul_id.rs, module
 * documentation): for every (token, slot) pair p = token*n_expert_used + slot,
 *     e = ids[p]
 *     out[p][col] = sum_{j<k} dequant(W[e][col][j]) * x[token][j]
 * with the sum taken in double, element by element in ascending j, and the
 * result rounded once to the output type.
 *
 * Storage read here, code by code, one bit at a time:
 *   * the packed row of (e, col) starts at byte (e*n + col) * row_bytes;
 *   * bit i of a row is bit (i mod 8) of byte floor(i/8) (little-endian u32
 *     words, codes least-significant-bit first);
 *   * affine 4/8-bit and codebook codes: 32/bits codes per u32 word, code j at
 *     word floor(j/(32/bits)), shift bits*(j mod (32/bits)); a 3-bit word keeps
 *     its top two bits unused (turboquant fast_switch_patch.py,
 *     _get_dequant_kernel: word = col / elems_per_u32,
 *     code = (word >> ((col % elems_per_u32) * bits)) & mask);
 *   * affine 6-bit: 4 codes per 3-byte triplet read as one little-endian 24-bit
 *     integer, code j at bit 6*(j mod 4) of triplet floor(j/4)
 *     (quantized_matmul_id.rs, expert_weight_bytes: "triplets_per_row");
 *   * NVFP4 and MXFP4: two E2M1 codes per byte, element 2i in the low nibble
 *     (spark_model helpers_a.rs: routed weights stored [N, K/2]).
 *
 * Dequantisation of code c in group g = floor(j / group_size):
 *   affine   : c * scale[e][col][g] + bias[e][col][g]          (bf16 scale and bias)
 *   codebook : codebook[c] * scale[e][col][g]                  (f16; fast_switch_patch.py
 *                                                              "cb[code] * scale")
 *   NVFP4    : e2m1(c) * e4m3(scale[e][col][floor(j/16)]) * scale2[e]
 *   MXFP4    : e2m1(c) * e8m0(scale[e][col][floor(j/32)])   (spark_model helpers_a.rs:
 *              native-MXFP4 routed experts carry one E8M0 scale per 32 values,
 *              [N, K/32]; no second-level scale)
 *
 * Out-of-range ids (e >= num_experts) produce an all-zero output row and are
 * counted in *bad_ids.
 *
 * Per-expert output bias (turboquant fast_switch_patch.py, the switch layer's
 * "y + mx.expand_dims(bias[indices], -2)"): oracle_add_expert_bias adds
 * bias[e][col] to the double result of every pair with a valid id, before the
 * single rounding to the output type; rows of out-of-range ids stay zero.
 *
 * Gated output (spark_model helpers_a.rs, MoeLayer: the fused gate+up kernel
 * with SiLU, or GELU for GeGLU experts after set_gelu_activation): with rows
 * [0, n/2) of each expert the gate and rows [n/2, n) the up projection,
 * oracle_glu_elems forms act(gate) * up in double from the double results
 * (bias already added), before the single rounding.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { O_FMT_AFFINE = 0, O_FMT_CODEBOOK = 1, O_FMT_NVFP4 = 2, O_FMT_MXFP4 = 3 };
enum { O_DT_F32 = 0, O_DT_BF16 = 1, O_DT_F16 = 2, O_DT_F64 = 3 /* oracle-only: x given exactly */ };

/* ---------------------------------------------------------------- decoders */

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double oracle_bf16_to_double(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 7) & 0xFF, f = h & 0x7F;
    double mag;
    if (e == 0xFF) return f ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0) mag = ldexp((double)f, -126 - 7);
    else mag = ldexp(1.0 + f / 128.0, e - 127);
    return s ? -mag : mag;
}

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_double(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double mag;
    if (e == 0x1F) return f ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0) mag = ldexp((double)f, -14 - 10);
    else mag = ldexp(1.0 + f / 1024.0, e - 15);
    return s ? -mag : mag;
}

/* OCP 8-bit floating point, E4M3 ("FN"): bias 7, no infinities, S.1111.111 is NaN,
 * exponent field 0 encodes subnormals f/8 * 2^-6. */
double oracle_e4m3_to_double(uint8_t b) {
    int s = (b >> 7) & 1, e = (b >> 3) & 0xF, f = b & 7;
    double mag;
    if (e == 0xF && f == 7) return NAN;
    if (e == 0) mag = ldexp((double)f, -6 - 3);
    else mag = ldexp(1.0 + f / 8.0, e - 7);
    return s ? -mag : mag;
}

/* OCP Microscaling E8M0 scale: an unsigned biased exponent, 2^(b - 127); 0xFF is NaN. */
double oracle_e8m0_to_double(uint8_t b) {
    if (b == 0xFF) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* OCP Microscaling FP4 E2M1: bias 1, no infinities or NaN, exponent field 0
 * encodes the subnormal f * 0.5. */
double oracle_e2m1_to_double(uint8_t c) {
    int s = (c >> 3) & 1, e = (c >> 1) & 3, f = c & 1;
    double mag;
    if (e == 0) mag = 0.5 * f;
    else mag = ldexp(1.0 + f / 2.0, e - 1);
    return s ? -mag : mag;
}

static double x_at(const void *x, int dt, uint64_t idx) {
    if (dt == O_DT_F64) return ((const double *)x)[idx];
    if (dt == O_DT_F32) return (double)((const float *)x)[idx];
    if (dt == O_DT_BF16) return oracle_bf16_to_double(((const uint16_t *)x)[idx]);
    return oracle_f16_to_double(((const uint16_t *)x)[idx]);
}

/* ------------------------------------------------------- rounding to storage */

/* Round v to the nearest value of a binary format with `mbits` fraction bits and
 * `ebits` exponent bits (IEEE layout, top exponent reserved for inf/NaN), ties
 * to even. Returns the bit pattern. */
static uint32_t round_to_binary(double v, int mbits, int ebits) {
    uint32_t sign = signbit(v) ? 1u : 0u;
    int bias = (1 << (ebits - 1)) - 1;
    int emin = 1 - bias, emax = bias;
    uint32_t inf_bits = ((1u << ebits) - 1u) << mbits;
    if (isnan(v)) return inf_bits | (1u << (mbits - 1));
    double a = fabs(v);
    if (a == 0.0) return sign << (ebits + mbits);
    if (isinf(a)) return (sign << (ebits + mbits)) | inf_bits;
    int ex;
    frexp(a, &ex);
    int E = ex - 1; /* 2^E <= a < 2^(E+1) */
    if (E < emin) E = emin;
    double q = ldexp(a, mbits - E); /* quantum of the binade becomes 1 */
    double r = nearbyint(q);        /* default rounding mode: nearest, ties to even */
    uint64_t ri = (uint64_t)r;
    if (ri >= (1ull << (mbits + 1))) { ri >>= 1; E += 1; }
    uint32_t bits;
    if (ri < (1ull << mbits)) {
        bits = (uint32_t)ri; /* subnormal */
    } else {
        if (E > emax) return (sign << (ebits + mbits)) | inf_bits;
        bits = ((uint32_t)(E + bias) << mbits) | (uint32_t)(ri - (1ull << mbits));
    }
    return (sign << (ebits + mbits)) | bits;
}

uint16_t oracle_double_to_bf16(double v) { return (uint16_t)round_to_binary(v, 7, 8); }
uint16_t oracle_double_to_f16(double v) { return (uint16_t)round_to_binary(v, 10, 5); }

/* Round n doubles to the output type: f32 (C conversion, nearest-even), bf16 or f16. */
void oracle_round_out(const double *in, void *out, uint64_t count, int out_dtype) {
    for (uint64_t i = 0; i < count; i++) {
        if (out_dtype == O_DT_F32) ((float *)out)[i] = (float)in[i];
        else if (out_dtype == O_DT_BF16) ((uint16_t *)out)[i] = oracle_double_to_bf16(in[i]);
        else ((uint16_t *)out)[i] = oracle_double_to_f16(in[i]);
    }
}

/* ------------------------------------------------------------ code storage */

uint64_t oracle_row_bytes(int fmt, int bits, uint32_t k) {
    if (fmt == O_FMT_NVFP4 || fmt == O_FMT_MXFP4) return (uint64_t)k / 2;
    if (fmt == O_FMT_AFFINE && bits == 6) return ((uint64_t)k + 3) / 4 * 3;
    uint32_t epw = 32u / (uint32_t)bits;
    return ((uint64_t)k + epw - 1) / epw * 4;
}

static unsigned bit_at(const uint8_t *row, uint64_t i) { return (row[i >> 3] >> (i & 7)) & 1u; }

/* Start bit of element j inside its packed row. */
static uint64_t code_start_bit(int fmt, int bits, uint32_t j) {
    if (fmt == O_FMT_NVFP4 || fmt == O_FMT_MXFP4) return 4ull * j;
    if (fmt == O_FMT_AFFINE && bits == 6) return 24ull * (j / 4) + 6ull * (j % 4);
    uint32_t epw = 32u / (uint32_t)bits;
    return 32ull * (j / epw) + (uint64_t)bits * (j % epw);
}

/* Code of element j of a packed row, read one bit at a time, least significant first. */
uint32_t oracle_code(const uint8_t *row, int fmt, int bits, uint32_t j) {
    uint64_t start = code_start_bit(fmt, bits, j);
    uint32_t c = 0;
    for (int b = 0; b < bits; b++) c |= (uint32_t)bit_at(row, start + (uint64_t)b) << b;
    return c;
}

/* ------------------------------------------------------------------ problem */

typedef struct {
    const void *x;
    const uint32_t *ids;
    const uint8_t *packed;
    const void *scales;
    const void *aux;
    uint32_t m, k, n, group_size, bits, n_expert_used, num_experts;
    int fmt, x_dtype;
    uint64_t row_bytes, groups;
} problem_t;

static double weight(const problem_t *P, uint32_t e, uint32_t col, uint32_t j) {
    uint64_t row_index = (uint64_t)e * P->n + col;
    const uint8_t *row = P->packed + row_index * P->row_bytes;
    uint32_t c = oracle_code(row, P->fmt, (int)P->bits, j);
    uint64_t sidx = row_index * P->groups + j / P->group_size;
    if (P->fmt == O_FMT_AFFINE) {
        double s = oracle_bf16_to_double(((const uint16_t *)P->scales)[sidx]);
        double b = oracle_bf16_to_double(((const uint16_t *)P->aux)[sidx]);
        return (double)c * s + b;
    }
    if (P->fmt == O_FMT_CODEBOOK) {
        double cb = oracle_f16_to_double(((const uint16_t *)P->aux)[c]);
        double s = oracle_f16_to_double(((const uint16_t *)P->scales)[sidx]);
        return cb * s;
    }
    if (P->fmt == O_FMT_MXFP4)
        return oracle_e2m1_to_double((uint8_t)c) * oracle_e8m0_to_double(((const uint8_t *)P->scales)[sidx]);
    /* NVFP4 */
    double s = oracle_e4m3_to_double(((const uint8_t *)P->scales)[sidx]);
    double s2 = (double)((const float *)P->aux)[e];
    return oracle_e2m1_to_double((uint8_t)c) * s * s2;
}

/* One output element: out[p][col]. Returns 0 and counts nothing for bad ids here. */
static double element(const problem_t *P, uint64_t p, uint32_t col) {
    uint32_t e = P->ids[p];
    if (e >= P->num_experts) return 0.0;
    uint64_t t = p / P->n_expert_used;
    double acc = 0.0;
    for (uint32_t j = 0; j < P->k; j++)
        acc += weight(P, e, col, j) * x_at(P->x, P->x_dtype, t * P->k + j);
    return acc;
}

typedef struct {
    const problem_t *P;
    double *out;
    const uint32_t *sp, *sc; /* sample mode: pair and column lists */
    uint64_t begin, end;     /* pair range (full mode) or sample range */
    int sample_mode;
} job_t;

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    const problem_t *P = J->P;
    if (J->sample_mode) {
        for (uint64_t i = J->begin; i < J->end; i++) J->out[i] = element(P, J->sp[i], J->sc[i]);
    } else {
        for (uint64_t p = J->begin; p < J->end; p++)
            for (uint32_t col = 0; col < P->n; col++) J->out[p * P->n + col] = element(P, p, col);
    }
    return NULL;
}

static int run_jobs(const problem_t *P, double *out, const uint32_t *sp, const uint32_t *sc,
                    uint64_t count, int sample_mode, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if ((uint64_t)nthreads > count) nthreads = count ? (int)count : 1;
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
    if (!th || !jobs) { free(th); free(jobs); return -1; }
    for (int i = 0; i < nthreads; i++) {
        jobs[i].P = P; jobs[i].out = out; jobs[i].sp = sp; jobs[i].sc = sc;
        jobs[i].sample_mode = sample_mode;
        jobs[i].begin = count * (uint64_t)i / (uint64_t)nthreads;
        jobs[i].end = count * (uint64_t)(i + 1) / (uint64_t)nthreads;
    }
    int rc = 0;
    int started = 0;
    for (int i = 1; i < nthreads; i++) {
        if (pthread_create(&th[i], NULL, worker, &jobs[i]) != 0) { rc = -1; break; }
        started = i;
    }
    worker(&jobs[0]);
    for (int i = 1; i <= started; i++) pthread_join(th[i], NULL);
    if (rc != 0) /* finish the ranges whose threads did not start */
        for (int i = started + 1; i < nthreads; i++) worker(&jobs[i]);
    free(th); free(jobs);
    return 0;
}

static int make_problem(problem_t *P, const void *x, const uint32_t *ids, const uint8_t *packed,
                        const void *scales, const void *aux, uint32_t m, uint32_t k, uint32_t n,
                        uint32_t group_size, uint32_t bits, int fmt, uint32_t n_expert_used,
                        uint32_t num_experts, int x_dtype) {
    if (!m || !k || !n || !group_size || !n_expert_used || !num_experts) return -1;
    if (fmt == O_FMT_AFFINE && bits != 4 && bits != 6 && bits != 8) return -1;
    if (fmt == O_FMT_CODEBOOK && bits != 2 && bits != 3 && bits != 4) return -1;
    if (fmt == O_FMT_NVFP4 && (bits != 4 || group_size != 16 || (k & 1))) return -1;
    if (fmt == O_FMT_MXFP4 && (bits != 4 || group_size != 32 || (k & 1))) return -1;
    if (fmt < 0 || fmt > 3 || x_dtype < 0 || x_dtype > 3) return -1;
    P->x = x; P->ids = ids; P->packed = packed; P->scales = scales; P->aux = aux;
    P->m = m; P->k = k; P->n = n; P->group_size = group_size; P->bits = bits;
    P->n_expert_used = n_expert_used; P->num_experts = num_experts;
    P->fmt = fmt; P->x_dtype = x_dtype;
    P->row_bytes = oracle_row_bytes(fmt, (int)bits, k);
    P->groups = ((uint64_t)k + group_size - 1) / group_size;
    return 0;
}

/* Full output [m*n_expert_used][n] in double. Returns -1 on invalid scalars,
 * otherwise the number of (token, slot) pairs whose id was out of range. */
int64_t oracle_qmm_id(const void *x, const uint32_t *ids, const uint8_t *packed,
                      const void *scales, const void *aux, double *out, uint32_t m, uint32_t k,
                      uint32_t n, uint32_t group_size, uint32_t bits, int fmt,
                      uint32_t n_expert_used, uint32_t num_experts, int x_dtype, int nthreads) {
    problem_t P;
    if (make_problem(&P, x, ids, packed, scales, aux, m, k, n, group_size, bits, fmt,
                     n_expert_used, num_experts, x_dtype))
        return -1;
    uint64_t R = (uint64_t)m * n_expert_used;
    if (run_jobs(&P, out, NULL, NULL, R, 0, nthreads)) return -1;
    int64_t bad = 0;
    for (uint64_t p = 0; p < R; p++) bad += ids[p] >= num_experts;
    return bad;
}

/* Selected elements out[sample_p[i]][sample_col[i]], i < count, in double. */
int oracle_qmm_id_sample(const void *x, const uint32_t *ids, const uint8_t *packed,
                         const void *scales, const void *aux, const uint32_t *sample_p,
                         const uint32_t *sample_col, uint64_t count, double *out_vals, uint32_t m,
                         uint32_t k, uint32_t n, uint32_t group_size, uint32_t bits, int fmt,
                         uint32_t n_expert_used, uint32_t num_experts, int x_dtype, int nthreads) {
    problem_t P;
    if (make_problem(&P, x, ids, packed, scales, aux, m, k, n, group_size, bits, fmt,
                     n_expert_used, num_experts, x_dtype))
        return -1;
    uint64_t R = (uint64_t)m * n_expert_used;
    for (uint64_t i = 0; i < count; i++)
        if (sample_p[i] >= R || sample_col[i] >= n) return -1;
    return run_jobs(&P, out_vals, sample_p, sample_col, count, 1, nthreads);
}

/* Maximum |w| over expert e's dequantised weights (for the per-element tolerance). */
double oracle_expert_max_abs_weight(const uint8_t *packed, const void *scales, const void *aux,
                                    uint32_t e, uint32_t k, uint32_t n, uint32_t group_size,
                                    uint32_t bits, int fmt, uint32_t num_experts) {
    problem_t P;
    if (make_problem(&P, NULL, NULL, packed, scales, aux, 1, k, n, group_size, bits, fmt, 1,
                     num_experts, O_DT_F32) || e >= num_experts)
        return -1.0;
    double mx = 0.0;
    for (uint32_t col = 0; col < n; col++)
        for (uint32_t j = 0; j < k; j++) {
            double w = fabs(weight(&P, e, col, j));
            if (w > mx) mx = w;
        }
    return mx;
}

/* ----------------------------------------------------------------- routing */

/* Routing of the R = m*n_expert_used pairs into per-expert groups.
 *   counts[e]       e < E: pairs with ids[p] == e;  counts[E]: pairs with an
 *                   out-of-range id.
 *   offsets[0..E+1] exclusive prefix sum of counts (offsets[E+1] == R).
 *   sorted_pairs[R] pair indices grouped by bucket in ascending bucket order
 *                   (experts 0..E-1, then the out-of-range bucket), ascending p
 *                   inside a bucket.
 *   tiles[2*i], tiles[2*i+1] = (expert, first row) of the i-th tile of
 *                   tile_rows consecutive rows, experts ascending, rows ascending.
 * Returns the number of tiles, or -1 if it would exceed max_tiles. */
int64_t oracle_route(const uint32_t *ids, uint64_t R, uint32_t E, uint32_t tile_rows,
                     uint32_t *counts, uint32_t *offsets, uint32_t *sorted_pairs, uint32_t *tiles,
                     uint64_t max_tiles) {
    for (uint32_t e = 0; e <= E; e++) counts[e] = 0;
    for (uint64_t p = 0; p < R; p++) counts[ids[p] < E ? ids[p] : E]++;
    offsets[0] = 0;
    for (uint32_t e = 0; e <= E; e++) offsets[e + 1] = offsets[e] + counts[e];
    uint64_t w = 0;
    for (uint32_t b = 0; b <= E; b++)
        for (uint64_t p = 0; p < R; p++) {
            uint32_t bucket = ids[p] < E ? ids[p] : E;
            if (bucket == b) sorted_pairs[w++] = (uint32_t)p;
        }
    uint64_t nt = 0;
    for (uint32_t e = 0; e < E; e++)
        for (uint32_t r0 = 0; r0 < counts[e]; r0 += tile_rows) {
            if (nt >= max_tiles) return -1;
            tiles[2 * nt] = e;
            tiles[2 * nt + 1] = r0;
            nt++;
        }
    return (int64_t)nt;
}

/* vals[i] += bias[e][col] for element i = (pair p, column col) with e = ids[p] <
 * num_experts (bias [num_experts, n], dtype 0 f32, 1 bf16, 2 f16). With pairs and
 * cols NULL, element i is pair i / n, column i % n. */
void oracle_add_expert_bias(double *vals, const uint32_t *pairs, const uint32_t *cols, uint64_t count,
                            const uint32_t *ids, const void *bias, int bias_dtype, uint32_t n,
                            uint32_t num_experts) {
    for (uint64_t i = 0; i < count; i++) {
        const uint64_t p = pairs ? pairs[i] : i / n;
        const uint64_t col = cols ? cols[i] : i % n;
        const uint32_t e = ids[p];
        if (e < num_experts) vals[i] += x_at(bias, bias_dtype, (uint64_t)e * n + col);
    }
}

/* act(g) in double: 0 SiLU, g / (1 + e^-g); 1 GELU in its tanh form,
 * g/2 (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))); 2 GELU in its erf form,
 * g/2 (1 + erf(g / sqrt(2))) = g * Phi(g). Other codes return NAN. */
double oracle_act(int act, double g) {
    if (act == 0) return g / (1.0 + exp(-g));
    if (act == 1) return 0.5 * g * (1.0 + tanh(sqrt(2.0 / 3.14159265358979323846) * (g + 0.044715 * g * g * g)));
    if (act == 2) return 0.5 * g * (1.0 + erf(g / sqrt(2.0)));
    return NAN;
}

/* out[i] = act(gate[i]) * up[i] for i < count. */
void oracle_glu_elems(const double *gate, const double *up, uint64_t count, int act, double *out) {
    for (uint64_t i = 0; i < count; i++) out[i] = oracle_act(act, gate[i]) * up[i];
}

/* ------------------------------------------- W4A4: NVFP4 activation quantisation
 *
 * The pages quantise weights to NVFP4 (E2M1 codes, one E4M3 scale per 16 values,
 * a second-level f32 scale; spark_model helpers_a.rs) and name a grouped NVFP4
 * GEMM whose activations are NVFP4 too (metrale helpers_b.rs,
 * build_cutlass_grouped_sfb: per-expert swizzled scale tables for that path), but
 * they do not say how activations are quantised. The reading here, per token t
 * (one row of x), with every step in f32 as a GPU kernel would take it:
 *   a   = max_j |x[t][j]|
 *   g   = a / 2688   (2688 = 448 * 6: the largest E4M3 scale times the largest
 *                     E2M1 value), or 0 when a = 0
 *   per block b of 16 values (k a multiple of 16):
 *     s_b  = E4M3(max_{j in b} |x[t][j]| / (6 * g)), nearest, ties to even,
 *            values above 448 taken as 448; 0 when g = 0
 *     d    = e4m3(s_b) * g
 *     q_j  = E2M1(x[t][j] / d), nearest, ties to even, magnitudes above 6 taken
 *            as 6, the sign of the quotient kept; code 0 when d = 0
 *   x^[t][j] = e2m1(q_j) * e4m3(s_b) * g   (in double: exact)
 * The matmul then takes x^ in place of x (oracle_qmm_id with O_DT_F64). */

static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Nearest E2M1 code of v (ties to the even code, |v| > 6 saturates to 6). The
 * magnitude codes 0..7 are in increasing order; "even" is the code's low bit. */
uint8_t oracle_e2m1_rne(float v) {
    uint8_t sign = signbit(v) ? 8u : 0u;
    double a = fabs((double)v);
    if (a >= 6.0) return (uint8_t)(sign | 7u);  /* saturate (also where far-off distances tie) */
    int best = 0;
    for (int c = 1; c < 8; c++) {
        double dc = fabs(E2M1_MAG[c] - a), db = fabs(E2M1_MAG[best] - a);
        if (dc < db || (dc == db && (c & 1) == 0)) best = c;
    }
    return (uint8_t)(sign | (uint8_t)best);
}

/* Nearest finite E4M3 code of v >= 0 (ties to the even code, values above 448
 * saturate to 448), by scanning the 127 non-negative finite codes in order. */
uint8_t oracle_e4m3_rne_satfinite(float v) {
    double a = (double)v;
    if (!(a > 0.0)) return 0u;
    if (a >= 448.0) return 0x7Eu;  /* saturate */
    int best = 0;
    for (int c = 1; c <= 0x7E; c++) {
        double dc = fabs(oracle_e4m3_to_double((uint8_t)c) - a);
        double db = fabs(oracle_e4m3_to_double((uint8_t)best) - a);
        if (dc < db || (dc == db && (c & 1) == 0)) best = c;
    }
    return (uint8_t)best;
}

/* Quantise x [m, k] (x_dtype) per the reading above. Any output may be NULL:
 * codes [m, k/2] (element 2i in the low nibble), scales [m, k/16] E4M3 bytes,
 * gscale [m] f32, xhat [m, k] double. Returns -1 when k is not a multiple of 16. */
int oracle_quantize_act_nvfp4(const void *x, int x_dtype, uint32_t m, uint32_t k, uint8_t *codes,
                              uint8_t *scales, float *gscale, double *xhat) {
    if (k == 0 || k % 16u != 0 || x_dtype < 0 || x_dtype > 2) return -1;
    for (uint32_t t = 0; t < m; t++) {
        float a = 0.0f;
        for (uint32_t j = 0; j < k; j++) {
            float v = fabsf((float)x_at(x, x_dtype, (uint64_t)t * k + j));
            if (v > a) a = v;
        }
        volatile float g = a / 2688.0f;  /* f32 division, no contraction */
        if (gscale) gscale[t] = g;
        for (uint32_t b = 0; b < k / 16u; b++) {
            float ab = 0.0f;
            for (uint32_t i = 0; i < 16; i++) {
                float v = fabsf((float)x_at(x, x_dtype, (uint64_t)t * k + 16u * b + i));
                if (v > ab) ab = v;
            }
            uint8_t s = 0;
            if (g > 0.0f) {
                volatile float six_g = 6.0f * g;
                volatile float q = ab / six_g;
                s = oracle_e4m3_rne_satfinite(q);
            }
            if (scales) scales[(uint64_t)t * (k / 16u) + b] = s;
            volatile float sv = (float)oracle_e4m3_to_double(s);
            volatile float d = sv * g;
            for (uint32_t i = 0; i < 16; i++) {
                uint64_t idx = (uint64_t)t * k + 16u * b + i;
                uint8_t c = 0;
                if (d > 0.0f) {
                    volatile float q = (float)x_at(x, x_dtype, idx) / d;
                    c = oracle_e2m1_rne(q);
                }
                if (codes) {
                    uint8_t *byte = codes + idx / 2;
                    if (idx % 2 == 0) *byte = (uint8_t)((*byte & 0xF0u) | c);
                    else *byte = (uint8_t)((*byte & 0x0Fu) | (uint8_t)(c << 4));
                }
                if (xhat) xhat[idx] = oracle_e2m1_to_double(c) * (double)sv * (double)g;
            }
        }
    }
    return 0;
}
