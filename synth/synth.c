/*
 * Seeded, counter-based synthetic input generator.
 *
 * This module produces the workload tensors (partial attention outputs and
 * softmax statistics) that both the CUDA path and the CPU oracle consume. It
 * holds none of the method's arithmetic: no LSE, no packing, no combine. Every
 * value is a pure function of (seed, tensor id, flat element index), so any
 * element of a multi-gigabyte tensor can be regenerated on its own, in any
 * order, on any number of threads, with identical bits.
 *
 * Random bits: the SplitMix64 generator (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014; the finaliser
 * constants are the ones Vigna published with his splitmix64.c). The i-th
 * output of a SplitMix64 stream started at state k is mix(k + (i + 1) * gamma);
 * a tensor's stream state k is itself derived from (seed, tensor id) by mixing.
 *
 * Distributions:
 *   uniform      a + (b - a) * u,           u in [0, 1) with 53 random bits
 *   loguniform   exp(ln a + (ln b - ln a) u)
 *   normal       Box-Muller (Box and Muller 1958): element pair p uses draws
 *                2p and 2p+1; even elements take the cosine branch, odd ones
 *                the sine branch.
 *   unit         u itself, as float64 (used for masks and categorical picks)
 *
 * Output formats: float32, float64, and the raw bits of bfloat16 or IEEE
 * binary16, rounded to nearest-even from the float64 value.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t stream_state(uint64_t seed, uint64_t tid)
{
    return mix64(mix64(seed + GAMMA) ^ (tid * 0xD1B54A32D192ED03ull + 1u));
}

static inline uint64_t draw(uint64_t state, uint64_t i)
{
    return mix64(state + (i + 1u) * GAMMA);
}

/* [0, 1) */
static inline double unit_closed_open(uint64_t x) { return (double)(x >> 11) * 0x1p-53; }
/* (0, 1): safe for log() */
static inline double unit_open(uint64_t x) { return ((double)(x >> 11) + 0.5) * 0x1p-53; }

/* Round a float64 to a binary format with `man` stored mantissa bits and
 * exponent bias `bias` (bfloat16: 7, 127; binary16: 10, 15); ties to even. */
static uint16_t round_to_16bit(double x, int man, int bias)
{
    const int exp_all_ones = 2 * bias + 1;
    uint16_t sign = signbit(x) ? (uint16_t)(1u << 15) : 0;
    if (isnan(x))
        return (uint16_t)(sign | (exp_all_ones << man) | (1u << (man - 1)));
    double a = fabs(x);
    if (isinf(a))
        return (uint16_t)(sign | (exp_all_ones << man));
    if (a == 0.0)
        return sign;
    int e = ilogb(a);
    const int emin = 1 - bias;
    if (e < emin)
        e = emin;
    double q = ldexp(1.0, e - man);     /* spacing of representable values */
    double m = nearbyint(a / q);        /* default rounding mode: nearest-even */
    if (m >= ldexp(1.0, man + 1)) {     /* rounded up into the next binade */
        m *= 0.5;
        e += 1;
    }
    if (e > bias)
        return (uint16_t)(sign | (exp_all_ones << man));
    if (m < ldexp(1.0, man))            /* subnormal: exponent field 0 */
        return (uint16_t)(sign | (uint16_t)m);
    return (uint16_t)(sign | ((uint16_t)(e + bias) << man) | (uint16_t)(m - ldexp(1.0, man)));
}

enum { DIST_NORMAL = 0, DIST_UNIFORM = 1, DIST_LOGUNIFORM = 2, DIST_UNIT = 3 };
enum { FMT_F32 = 0, FMT_BF16 = 1, FMT_F16 = 2, FMT_F64 = 3 };

static inline double value_at(uint64_t st, int dist, double p0, double p1, uint64_t i)
{
    switch (dist) {
    case DIST_NORMAL: {
        uint64_t p = i >> 1;
        double r = sqrt(-2.0 * log(unit_open(draw(st, 2 * p))));
        double th = 6.283185307179586 * unit_closed_open(draw(st, 2 * p + 1));
        return p0 + p1 * ((i & 1) ? r * sin(th) : r * cos(th));
    }
    case DIST_UNIFORM:
        return p0 + (p1 - p0) * unit_closed_open(draw(st, i));
    case DIST_LOGUNIFORM: {
        double la = log(p0), lb = log(p1);
        return exp(la + (lb - la) * unit_closed_open(draw(st, i)));
    }
    default:
        return unit_closed_open(draw(st, i));
    }
}

static inline void store(void* out, uint64_t k, int fmt, double v)
{
    switch (fmt) {
    case FMT_F32: ((float*)out)[k] = (float)v; break;
    case FMT_BF16: ((uint16_t*)out)[k] = round_to_16bit(v, 7, 127); break;
    case FMT_F16: ((uint16_t*)out)[k] = round_to_16bit(v, 10, 15); break;
    default: ((double*)out)[k] = v; break;
    }
}

/*
 * Fill out[k] for k < n with element index (idx ? idx[k] : start + k) of the
 * stream (seed, tid) under distribution `dist` with parameters p0, p1.
 */
void synth_fill(uint64_t seed, uint64_t tid, int dist, double p0, double p1, uint64_t start,
                const uint64_t* idx, int64_t n, int fmt, void* out)
{
    const uint64_t st = stream_state(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k) {
        uint64_t i = idx ? idx[k] : start + (uint64_t)k;
        store(out, (uint64_t)k, fmt, value_at(st, dist, p0, p1, i));
    }
}

/* Raw 64-bit draw, for the generator's own tests. */
uint64_t synth_raw(uint64_t seed, uint64_t tid, uint64_t i)
{
    return draw(stream_state(seed, tid), i);
}

/* The rounding used for bfloat16 / binary16 outputs, exposed for tests. */
uint16_t synth_round16(double x, int fmt)
{
    return fmt == FMT_BF16 ? round_to_16bit(x, 7, 127) : round_to_16bit(x, 10, 15);
}
