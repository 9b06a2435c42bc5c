/*
 * CPU oracle for the decode-context-parallel (DCP) attention exchange and the
 * Ulysses sequence/head layout transforms.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline / reference leg may load this library. The product path never
 * calls it and shares no code with it: it has its own payload decoding, its
 * own rounding, its own index arithmetic. Everything is plain loops in
 * float64, in the order the method states, so that it can be checked by eye
 * against the sources cited on each function.
 *
 * Sources (titles of the pages that define the operations):
 *  [DCP]  vLLM-Ascend pull request "[Performance][Attention] Fuse local SFA LSE
 *         formation into DCP pack": section "What this PR does / why we need
 *         it?" (the Before/After pipelines and the invalid-statistic rule) and
 *         "How was this patch tested?" (scatter_dim 0 and 1, strided inputs).
 *  [ULY]  FastVideo compare view "[perf] Probe H3 chunked all-to-all with direct
 *         output slices": the all_to_all_4D(x, 2, 1) / (x, 1, 2) operand shapes
 *         [B, S/W, H, D] <-> [B, S, H/W, D] in benchmark_ulysses_a2a.py and
 *         probe_ulysses_launch.py, with byte-identical parity to the NCCL path.
 *  The combine formula itself is not printed on the pages (the pull request
 *  reuses a stable combine it already had); the oracle uses the standard log-sum-exp merge of
 *  partial softmax results: LSE* = logsumexp_r LSE_r, O = sum_r exp(LSE_r - LSE*) O_r,
 *  with -inf contributions weighted zero and an all-invalid row giving O = 0,
 *  LSE = -inf.
 *
 * Layouts (row-major, last index fastest; W ranks, T tokens, H heads, Hc = H/W):
 *   O        [W][T][H][D]  payload (bf16 or fp16 bits), element strides given
 *   max, sum [W][T][H]     float32, element strides given
 *   packet   scatter_dim 1: pkt_o [W_src][W_dst][T][Hc][D], pkt_lse [W_src][W_dst][T][Hc]
 *            scatter_dim 0: pkt_o [W_src][W_dst][T/W][H][D], pkt_lse [W_src][W_dst][T/W][H]
 *   received recv[dst][src] = pkt[src][dst]
 *   combined out [W_dst][N][D], out_lse [W_dst][N], N = rows per block
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_BF16 = 0, ORACLE_FP16 = 1 };

/* Threads of the parallel loops below (the benchmark times the oracle on all
 * host cores and on one). oracle_set_threads returns the count now in effect. */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
    return oracle_threads();
}

/* ------------------------------------------------------------------------- */
/* payload formats, from their bit-level definitions                          */

/* bfloat16 is the upper half of an IEEE binary32. */
static double bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double fp16_value(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int ex = (b >> 10) & 0x1f;
    int fr = b & 0x3ff;
    double v;
    if (ex == 0)
        v = ldexp((double)fr, -24);                 /* zero or subnormal */
    else if (ex == 31)
        v = fr ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + fr), ex - 25);
    return sign ? -v : v;
}

static double payload_value(uint16_t b, int dtype)
{
    return dtype == ORACLE_BF16 ? bf16_value(b) : fp16_value(b);
}

/* Nearest-even rounding of a float64 to a 16-bit format with `man` fraction
 * bits and exponent bias `bias`: the value is snapped to the spacing of its
 * binade (or of the subnormal range), with overflow to infinity. */
static uint16_t round_16(double x, int man, int bias)
{
    int top = 2 * bias + 1;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x))
        return (uint16_t)(sign | (top << man) | (1 << (man - 1)));
    double a = fabs(x);
    if (isinf(a))
        return (uint16_t)(sign | (top << man));
    if (a == 0.0)
        return sign;
    int e = ilogb(a);
    if (e < 1 - bias)
        e = 1 - bias;
    double spacing = ldexp(1.0, e - man);
    double q = nearbyint(a / spacing);
    if (q >= ldexp(1.0, man + 1)) {
        q /= 2;
        e += 1;
    }
    if (e > bias)
        return (uint16_t)(sign | (top << man));
    if (q < ldexp(1.0, man))
        return (uint16_t)(sign | (uint16_t)q);
    return (uint16_t)(sign | ((e + bias) << man) | (uint16_t)(q - ldexp(1.0, man)));
}

static uint16_t payload_round(double x, int dtype)
{
    return dtype == ORACLE_BF16 ? round_16(x, 7, 127) : round_16(x, 10, 15);
}

double oracle_payload_value(uint16_t b, int dtype) { return payload_value(b, dtype); }
uint16_t oracle_payload_round(double x, int dtype) { return payload_round(x, dtype); }

/* ------------------------------------------------------------------------- */
/* [DCP] LSE formation. LSE = softmax_max + log(softmax_sum); a non-finite max,
 * a non-finite sum, or a sum <= 0 is an invalid statistic and gives -inf.    */

double oracle_lse(double m, double s)
{
    if (!isfinite(m) || !isfinite(s) || !(s > 0.0))
        return -INFINITY;
    return m + log(s);
}

/* ------------------------------------------------------------------------- */
/* [DCP] pack: the send packet, partial outputs in one region and LSE in the
 * other, destination-major per source rank.
 *   scatter_dim 1 (head chunks):  pkt[r][j][t][hc]  = row (t, j*Hc + hc) of rank r
 *   scatter_dim 0 (token chunks): pkt[r][j][tc][h]  = row (j*Tc + tc, h) of rank r
 * Payload bits are copied unchanged. pkt_lse32 receives LSE rounded to float32
 * (the packet's LSE type); pkt_lse64 the unrounded value. Either may be NULL. */

void oracle_pack(const uint16_t* o, int64_t so_r, int64_t so_t, int64_t so_h,
                 const float* mx, int64_t sm_r, int64_t sm_t, int64_t sm_h,
                 const float* sm, int64_t ss_r, int64_t ss_t, int64_t ss_h,
                 int W, int64_t T, int64_t H, int64_t D, int scatter_dim,
                 uint16_t* pkt_o, float* pkt_lse32, double* pkt_lse64)
{
    int64_t Hc = H / W, Tc = T / W;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int r = 0; r < W; ++r) {
            for (int64_t h = 0; h < H; ++h) {
                int64_t j, slot; /* destination rank and packet row within pkt[r][j] */
                if (scatter_dim == 1) {
                    j = h / Hc;
                    slot = t * Hc + (h % Hc);
                } else {
                    j = t / Tc;
                    slot = (t % Tc) * H + h;
                }
                int64_t rows_per_block = T * Hc; /* equals Tc * H */
                int64_t dst_row = ((int64_t)r * W + j) * rows_per_block + slot;
                const uint16_t* src = o + r * so_r + t * so_t + h * so_h;
                for (int64_t d = 0; d < D; ++d)
                    pkt_o[dst_row * D + d] = src[d];
                double lse = oracle_lse((double)mx[r * sm_r + t * sm_t + h * sm_h],
                                        (double)sm[r * ss_r + t * ss_t + h * ss_h]);
                if (pkt_lse32)
                    pkt_lse32[dst_row] = (float)lse;
                if (pkt_lse64)
                    pkt_lse64[dst_row] = lse;
            }
        }
    }
}

/* [DCP] the Before pipeline's pack: LSE was materialized first as its own
 * tensor lse [W][T][H] (element strides given); a rearranging step moves it
 * into the packet's LSE region while the pack copies the payload. Same layout
 * as oracle_pack; the LSE values are copied bit for bit. */
void oracle_pack_from_lse(const uint16_t* o, int64_t so_r, int64_t so_t, int64_t so_h,
                          const float* lse, int64_t sl_r, int64_t sl_t, int64_t sl_h,
                          int W, int64_t T, int64_t H, int64_t D, int scatter_dim,
                          uint16_t* pkt_o, float* pkt_lse)
{
    int64_t Hc = H / W, Tc = T / W;
    for (int64_t t = 0; t < T; ++t)
        for (int r = 0; r < W; ++r)
            for (int64_t h = 0; h < H; ++h) {
                int64_t j, slot;
                if (scatter_dim == 1) {
                    j = h / Hc;
                    slot = t * Hc + (h % Hc);
                } else {
                    j = t / Tc;
                    slot = (t % Tc) * H + h;
                }
                int64_t dst_row = ((int64_t)r * W + j) * (T * Hc) + slot;
                const uint16_t* src = o + r * so_r + t * so_t + h * so_h;
                for (int64_t d = 0; d < D; ++d)
                    pkt_o[dst_row * D + d] = src[d];
                pkt_lse[dst_row] = lse[r * sl_r + t * sl_t + h * sl_h];
            }
}

/* ------------------------------------------------------------------------- */
/* [DCP] the all-to-all, emulated: W simulated ranks each hold W blocks, block
 * j of rank r goes to rank j and lands in slot r. recv[j][r] = send[r][j].   */

void oracle_permute(const uint8_t* send, uint8_t* recv, int W, int64_t block_bytes)
{
    for (int r = 0; r < W; ++r)
        for (int j = 0; j < W; ++j)
            memcpy(recv + ((int64_t)j * W + r) * block_bytes,
                   send + ((int64_t)r * W + j) * block_bytes, (size_t)block_bytes);
}

/* ------------------------------------------------------------------------- */
/* Stable log-sum-exp combine of one row from W contributions.
 *   o   [W][D] partial outputs, lse [W] their log-sum-exp statistics.
 * Contributions with lse = -inf (or NaN) are skipped, never multiplied by 0,
 * so their payload cannot reach the result. */

static void combine_row(int W, int64_t D, const double* o, const double* lse,
                        double* out, double* out_lse)
{
    int any = 0;
    double M = -INFINITY;
    for (int r = 0; r < W; ++r) {
        if (lse[r] > -INFINITY) {
            any = 1;
            if (lse[r] > M)
                M = lse[r];
        }
    }
    for (int64_t d = 0; d < D; ++d)
        out[d] = 0.0;
    if (!any) {
        *out_lse = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int r = 0; r < W; ++r)
        if (lse[r] > -INFINITY)
            sum += exp(lse[r] - M);
    double L = M + log(sum);
    for (int r = 0; r < W; ++r) {
        if (!(lse[r] > -INFINITY))
            continue;
        double w = exp(lse[r] - L);
        for (int64_t d = 0; d < D; ++d)
            out[d] += w * o[r * D + d];
    }
    *out_lse = L;
}

/* The combine on float64 partials: o [W][N][D], lse [W][N] -> out [N][D], out_lse [N]. */
void oracle_combine_f64(int W, int64_t N, int64_t D, const double* o, const double* lse,
                        double* out, double* out_lse)
{
#pragma omp parallel
    {
        double* orow = malloc(sizeof(double) * (size_t)(W * D));
        double* l = malloc(sizeof(double) * (size_t)W);
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            for (int r = 0; r < W; ++r) {
                l[r] = lse[r * N + n];
                for (int64_t d = 0; d < D; ++d)
                    orow[r * D + d] = o[(r * N + n) * D + d];
            }
            combine_row(W, D, orow, l, out + n * D, out_lse + n);
        }
        free(orow);
        free(l);
    }
}

/* The combine each destination rank runs on what it received:
 *   recv_o [W_dst][W_src][N][D] payload bits, recv_lse [W_dst][W_src][N] float32
 *   -> out [W_dst][N][D] (float64, unrounded), out_lse [W_dst][N],
 *      out_rounded (optional) the payload-dtype nearest-even rounding of out.   */
void oracle_combine(const uint16_t* recv_o, const float* recv_lse, int W, int64_t N, int64_t D,
                    int dtype, double* out, double* out_lse, uint16_t* out_rounded)
{
#pragma omp parallel
    {
        double* orow = malloc(sizeof(double) * (size_t)(W * D));
        double* l = malloc(sizeof(double) * (size_t)W);
#pragma omp for schedule(static)
        for (int64_t jn = 0; jn < (int64_t)W * N; ++jn) {
            int64_t j = jn / N, n = jn % N;
            for (int r = 0; r < W; ++r) {
                int64_t src_row = (j * W + r) * N + n;
                l[r] = (double)recv_lse[src_row];
                for (int64_t d = 0; d < D; ++d)
                    orow[r * D + d] = payload_value(recv_o[src_row * D + d], dtype);
            }
            combine_row(W, D, orow, l, out + jn * D, out_lse + jn);
            if (out_rounded)
                for (int64_t d = 0; d < D; ++d)
                    out_rounded[jn * D + d] = payload_round(out[jn * D + d], dtype);
        }
        free(orow);
        free(l);
    }
}

/* ------------------------------------------------------------------------- */
/* Pack -> all-to-all -> combine in one pass, straight from the definitions:
 * destination j's row (t, hc) merges row (t, h = j*Hc + hc) of every source
 * rank, with each LSE formed from that rank's max and sum (head scatter).
 *   out [W][T][Hc][D], out_lse [W][T][Hc]. */
void oracle_fused(const uint16_t* o, int64_t so_r, int64_t so_t, int64_t so_h,
                  const float* mx, int64_t sm_r, int64_t sm_t, int64_t sm_h,
                  const float* sm, int64_t ss_r, int64_t ss_t, int64_t ss_h,
                  int W, int64_t T, int64_t H, int64_t D, int dtype,
                  double* out, double* out_lse, uint16_t* out_rounded)
{
    int64_t Hc = H / W;
#pragma omp parallel
    {
        double* orow = malloc(sizeof(double) * (size_t)(W * D));
        double* l = malloc(sizeof(double) * (size_t)W);
#pragma omp for schedule(static)
        for (int64_t th = 0; th < T * H; ++th) {
            int64_t t = th / H, h = th % H;
            int64_t j = h / Hc, hc = h % Hc;
            for (int r = 0; r < W; ++r) {
                l[r] = oracle_lse((double)mx[r * sm_r + t * sm_t + h * sm_h],
                                  (double)sm[r * ss_r + t * ss_t + h * ss_h]);
                const uint16_t* src = o + r * so_r + t * so_t + h * so_h;
                for (int64_t d = 0; d < D; ++d)
                    orow[r * D + d] = payload_value(src[d], dtype);
            }
            int64_t dst_row = (j * T + t) * Hc + hc;
            combine_row(W, D, orow, l, out + dst_row * D, out_lse + dst_row);
            if (out_rounded)
                for (int64_t d = 0; d < D; ++d)
                    out_rounded[dst_row * D + d] = payload_round(out[dst_row * D + d], dtype);
        }
        free(orow);
        free(l);
    }
}

/* The same merge for an arbitrary list of rows gathered by the caller:
 * o [W][n][D] payload bits, max/sum [W][n] -> out [n][D], out_lse [n]. Used to
 * check sampled rows of full-size problems without materialising them. */
void oracle_fused_gathered(const uint16_t* o, const float* mx, const float* sm, int W, int64_t n,
                           int64_t D, int dtype, double* out, double* out_lse,
                           uint16_t* out_rounded)
{
#pragma omp parallel
    {
        double* orow = malloc(sizeof(double) * (size_t)(W * D));
        double* l = malloc(sizeof(double) * (size_t)W);
#pragma omp for schedule(static)
        for (int64_t k = 0; k < n; ++k) {
            for (int r = 0; r < W; ++r) {
                l[r] = oracle_lse((double)mx[r * n + k], (double)sm[r * n + k]);
                for (int64_t d = 0; d < D; ++d)
                    orow[r * D + d] = payload_value(o[(r * n + k) * D + d], dtype);
            }
            combine_row(W, D, orow, l, out + k * D, out_lse + k);
            if (out_rounded)
                for (int64_t d = 0; d < D; ++d)
                    out_rounded[k * D + d] = payload_round(out[k * D + d], dtype);
        }
        free(orow);
        free(l);
    }
}

/* ------------------------------------------------------------------------- */
/* [ULY] all_to_all_4D(x, scatter_dim=2, gather_dim=1): rank r holds
 * in[r] = [B][S_l][H][D]; its head chunk j goes to rank j, which concatenates
 * the chunks of ranks 0..W-1 along the sequence:
 *   out[j][b][r*S_l + s][hc] = in[r][b][s][j*Hc + hc]                          */
void oracle_seq2head(const uint8_t* in, uint8_t* out, int W, int64_t B, int64_t S_l, int64_t H,
                     int64_t D, int64_t elem_bytes)
{
    int64_t Hc = H / W, S = S_l * W, row = D * elem_bytes;
    for (int j = 0; j < W; ++j)
        for (int64_t b = 0; b < B; ++b)
            for (int r = 0; r < W; ++r)
                for (int64_t s = 0; s < S_l; ++s)
                    for (int64_t hc = 0; hc < Hc; ++hc) {
                        int64_t dst = (((int64_t)j * B + b) * S + (int64_t)r * S_l + s) * Hc + hc;
                        int64_t src = (((int64_t)r * B + b) * S_l + s) * H + (int64_t)j * Hc + hc;
                        memcpy(out + dst * row, in + src * row, (size_t)row);
                    }
}

/* [ULY] all_to_all_4D(x, scatter_dim=1, gather_dim=2), the inverse: rank r
 * holds in[r] = [B][S][Hc][D]; its sequence chunk j goes to rank j, which
 * concatenates the chunks of ranks 0..W-1 along the heads:
 *   out[j][b][s][r*Hc + hc] = in[r][b][j*S_l + s][hc]                          */
void oracle_head2seq(const uint8_t* in, uint8_t* out, int W, int64_t B, int64_t S_l, int64_t H,
                     int64_t D, int64_t elem_bytes)
{
    int64_t Hc = H / W, S = S_l * W, row = D * elem_bytes;
    for (int j = 0; j < W; ++j)
        for (int64_t b = 0; b < B; ++b)
            for (int64_t s = 0; s < S_l; ++s)
                for (int r = 0; r < W; ++r)
                    for (int64_t hc = 0; hc < Hc; ++hc) {
                        int64_t dst = (((int64_t)j * B + b) * S_l + s) * H + (int64_t)r * Hc + hc;
                        int64_t src = (((int64_t)r * B + b) * S + (int64_t)j * S_l + s) * Hc + hc;
                        memcpy(out + dst * row, in + src * row, (size_t)row);
                    }
}
