/*
 * Seeded synthetic inputs for the quantized-attention workloads.
 *
 * This file holds no arithmetic of the attention method.  It only draws the
 * BF16 activations that both the CPU oracle and the CUDA library consume:
 *   - a counter-based generator: splitmix64 (Steele, Lea and Flood, "Fast
 *     splittable pseudorandom number generators", OOPSLA 2014) keyed by
 *     (seed, stream) and indexed by the logical element index;
 *   - standard normals by the Box-Muller transform in FP64;
 *   - three value recipes: plain N(mean, std^2); N(0,1) plus a per-(h,d)
 *     offset; and per-(b,t,h) RMS normalisation times a per-(h,d) gamma.
 *
 * The logical element index of x[b,t,h,d] is ((b*T + t)*H + h)*D + d whatever
 * the memory layout, so every layout (separate [B,T,H,D] tensors or one packed
 * [B,T,3,H,D] buffer) holds the same values.  Because the generator is
 * counter-based the fill is order-free and runs in parallel.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t splitmix64(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint32_t stream) {
    return splitmix64(seed ^ ((uint64_t)stream * 0xD1B54A32D192ED03ull));
}

/* Standard normal number n of the (seed, stream) sequence.  Numbers 2p and
 * 2p+1 come from one Box-Muller pair built on uniforms 2p and 2p+1. */
static inline double normal_at(uint64_t key, uint64_t n) {
    uint64_t pair = n >> 1;
    double u1 = ((double)(splitmix64(key + 2 * pair) >> 11) + 1.0) * 0x1.0p-53; /* (0,1] */
    double u2 = (double)(splitmix64(key + 2 * pair + 1) >> 11) * 0x1.0p-53;     /* [0,1) */
    double r = sqrt(-2.0 * log(u1));
    double a = 6.283185307179586476925286766559 * u2;
    return (n & 1) ? r * sin(a) : r * cos(a);
}

/* float -> bfloat16 bits, round to nearest even (inputs here are finite). */
static inline uint16_t to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Fill n FP32 values with float(mean + std * z_i), i = 0..n-1. */
void synth_normal_f32(float* out, int64_t n, uint64_t seed, uint32_t stream,
                      double mean, double std) {
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(mean + std * normal_at(key, (uint64_t)i));
}

enum { SYNTH_NORMAL = 0, SYNTH_OFFSET = 1, SYNTH_RMSNORM = 2 };

/*
 * Fill a logical [B,T,H,D] BF16 tensor at `out` with element strides
 * (sb, st, sh) and unit stride along d.
 *   kind SYNTH_NORMAL : bf16(float(mean + std*z))
 *   kind SYNTH_OFFSET : bf16(float(z) + vec[h*D+d])            (vec = offset)
 *   kind SYNTH_RMSNORM: x = float(z); ms = mean_d x^2 (FP64);
 *                       inv = float(1/sqrt(ms + 1e-6));
 *                       bf16((x*inv) * vec[h*D+d])              (vec = gamma)
 */
void synth_fill_bf16(uint16_t* out, int B, int T, int H, int D,
                     int64_t sb, int64_t st, int64_t sh,
                     uint64_t seed, uint32_t stream, int kind,
                     double mean, double std, const float* vec) {
    uint64_t key = stream_key(seed, stream);
    int64_t rows = (int64_t)B * T * H;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t h = r % H, bt = r / H;
        int64_t t = bt % T, b = bt / T;
        uint16_t* dst = out + b * sb + t * st + h * sh;
        uint64_t base = (uint64_t)r * (uint64_t)D;
        if (kind == SYNTH_NORMAL) {
            for (int d = 0; d < D; ++d)
                dst[d] = to_bf16((float)(mean + std * normal_at(key, base + d)));
        } else if (kind == SYNTH_OFFSET) {
            for (int d = 0; d < D; ++d)
                dst[d] = to_bf16((float)normal_at(key, base + d) + vec[h * D + d]);
        } else {
            float x[1024];
            double ms = 0.0;
            for (int d = 0; d < D; ++d) {
                x[d] = (float)normal_at(key, base + d);
                ms += (double)x[d] * (double)x[d];
            }
            ms /= (double)D;
            float inv = (float)(1.0 / sqrt(ms + 1e-6));
            for (int d = 0; d < D; ++d) dst[d] = to_bf16((x[d] * inv) * vec[h * D + d]);
        }
    }
}
