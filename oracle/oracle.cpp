// CPU oracle for SageAttention-style quantized self-attention.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
// this file: only tests/, the smoke check and the benchmark's CPU-baseline arm
// use it.  It shares no code, header, table or constant generator with the CUDA
// library.
//
// It emulates, step by step and in the order the pages give, the numerical
// policy of the dense Sage-compatible attention described in
//   "H3 Performance Roadmap", Phase 4: Dense Sage-Compatible Attention
//     (keep Sage2's per-warp INT8 Q/K quantization, FP8 V, its accumulation and
//      K smoothing; consume strided BSHD; emit token-major output), and
//   "H3 Performance Roadmap", the Sage2 decomposition paragraphs (K smoothing,
//     Q/K INT8 quantization, V transpose + FP8 quantization, fused mainloop),
//   "Phase 2B Aligned Numerical Prototype", Exactness (the checkpoints:
//     INT32-to-FP32 QK scores, per-epoch online-softmax m and d, FP8 E4M3
//     probability words, FP32 rescale values, FP32 RO after every epoch, the
//     final reciprocal, final BF16 output) and Decision (K64 epochs).
//
// Where the pages are silent the plainest reading is taken (each is listed in
// the repository's design notes):
//   * Q scale per 32-token group, K scale per 64-token group, one FP32 scale per
//     group over all channels; symmetric, scale = amax/127, round to nearest even,
//     clamp to [-127, 127]; amax == 0 gives scale 0 and all-zero words.
//   * K smoothing subtracts the per-(b,h,channel) mean over all valid keys; the
//     mean is an FP64 sum, sequential within each 64-token chunk, then sequential
//     over chunks, divided by Tkv and rounded to FP32; the smoothed value stays
//     FP32 (no BF16 re-rounding).  Neither Q nor V is smoothed.
//   * V scale per (b,h,channel): sv = amax/448; v8 = e4m3(v * (448/amax)).
//   * Scores: t = float(acc) * ((sq*sk) * c), c = float(scale * log2(e)).
//   * Online softmax in the log2 domain per epoch of `epoch` keys; probabilities
//     p = exp2(t - m) in FP32, stored as e4m3(448 * p); d sums the FP32 p.
//   * RO <- RO*alpha + sum_j dec(p8_j)*dec(v8_jc), FP32, ascending j.
//   * out = bf16((RO * (1/d)) * (sv/448)).
//   * Optional Q/K RMSNorm + RoPE before quantization ("H3 Performance Roadmap",
//     Component 2 execution order item 1 and the strided-NHD paragraph: Q/K
//     normalization and RoPE applied where the attention consumes Q and K), see
//     orc_qk_norm_rope: the quantization then reads its BF16 result.
// Compiled with -ffp-contract=off so that no multiply-add is fused.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>
#include <limits>

namespace {

// ----------------------------------------------------------------------------
// Number formats, written from their definitions.
// bfloat16: the upper 16 bits of an IEEE binary32.
// FP8 E4M3 (OCP 8-bit floating point, "E4M3"): 1 sign bit, 4 exponent bits
// with bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN; the largest
// finite magnitude is 1.75 * 2^8 = 448; subnormals are m * 2^-9.
// ----------------------------------------------------------------------------
inline float bf16_decode(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// Round an IEEE binary32 to the nearest bfloat16, ties to even.
inline uint16_t bf16_encode(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);  // quiet NaN
    uint32_t upper = u >> 16, lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;  // carries into exponent
    return (uint16_t)upper;
}

inline float e4m3_decode(uint8_t b) {
    int s = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (e == 0xF && m == 7) return std::numeric_limits<float>::quiet_NaN();
    if (e == 0) v = std::ldexp((double)m, -9);
    else v = std::ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

// All 256 E4M3 values, decoded once by e4m3_decode (a lookup, not new arithmetic).
struct E4M3Table {
    float v[256];
    E4M3Table() { for (int i = 0; i < 256; ++i) v[i] = e4m3_decode((uint8_t)i); }
};
const E4M3Table& e4m3_table() {
    static const E4M3Table t;
    return t;
}

// Round half to even of a non-negative double to an integer-valued double.
inline double rne(double x) {
    double f = std::floor(x), r = x - f;
    if (r > 0.5) return f + 1;
    if (r < 0.5) return f;
    return (std::fmod(f, 2.0) == 0.0) ? f : f + 1;
}

// Nearest E4M3 value, ties to even; magnitudes beyond 448 saturate to 448.
inline uint8_t e4m3_encode(float x) {
    if (std::isnan(x)) return 0x7F;
    uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
    double a = std::fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    uint8_t code;
    if (a < std::ldexp(1.0, -6)) {
        // subnormal range: multiples of 2^-9; m == 8 is the smallest normal, code 0x08
        code = (uint8_t)rne(a * 512.0);
    } else {
        int e;
        double fr = std::frexp(a, &e);   // a = fr * 2^e, fr in [0.5, 1)
        int E = e - 1;                   // a = (2*fr) * 2^E, 2*fr in [1, 2)
        double m = rne((2.0 * fr - 1.0) * 8.0);
        if (m == 8.0) { m = 0; E += 1; }
        int biased = E + 7;
        code = (uint8_t)((biased << 3) | (int)m);
        if (code > 0x7E) code = 0x7E;
    }
    return sign | code;
}

// Symmetric INT8 quantization of one value with a precomputed inverse step.
inline int8_t quant_i8(float x, float inv) {
    float y = x * inv;                          // FP32 product, round to nearest
    double r = std::nearbyint((double)y);       // ties to even (default rounding mode)
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return (int8_t)r;
}

const int KMEAN_CHUNK = 64;
const double LOG2E = 1.44269504088896340736;

}  // namespace

extern "C" {

// ---------------------------------------------------------------- codecs ----
float orc_bf16_decode(uint16_t h) { return bf16_decode(h); }
uint16_t orc_bf16_encode(float f) { return bf16_encode(f); }
float orc_e4m3_decode(uint8_t b) { return e4m3_decode(b); }
uint8_t orc_e4m3_encode(float f) { return e4m3_encode(f); }

void orc_bf16_encode_array(const float* x, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_encode(x[i]);
}
void orc_e4m3_encode_array(const float* x, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(x[i]);
}

// The log2-domain softmax constant c = float(scale * log2(e)).
float orc_log2_scale(float scale) { return (float)((double)scale * LOG2E); }

// ------------------------------------------------------------ quantize ------
// Q, K, V are BF16 bit patterns viewed as [B, T, H, D] with element strides
// (sb, st, sh) and unit stride along d.  Outputs (all dense, natural order):
//   km [B,H,D]  f32   K channel means
//   sq [B,H,ceil(Tq/gq)]  f32   Q group scales
//   sk [B,H,ceil(Tkv/gk)] f32   K group scales
//   sv [B,H,D]  f32   V channel scales (amax/448)
//   q8 [B,H,Tq,D] i8, k8 [B,H,Tkv,D] i8, v8 [B,H,Tkv,D] e4m3 bytes
// Returns 0, or -1 on a bad argument.
int orc_quantize(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 int64_t q_sb, int64_t q_st, int64_t q_sh,
                 int64_t k_sb, int64_t k_st, int64_t k_sh,
                 int64_t v_sb, int64_t v_st, int64_t v_sh,
                 int B, int Tq, int Tkv, int H, int D, int gq, int gk,
                 float* km, float* sq, float* sk, float* sv,
                 int8_t* q8, int8_t* k8, uint8_t* v8) {
    if (B < 1 || Tq < 1 || Tkv < 1 || H < 1 || D < 1 || gq < 1 || gk < 1) return -1;
    const int nq = (Tq + gq - 1) / gq, nk = (Tkv + gk - 1) / gk;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const int64_t bh = (int64_t)b * H + h;
            // K smoothing statistics: FP64 chunk sums in token order, then chunks in order.
            std::vector<double> total(D, 0.0);
            for (int c0 = 0; c0 < Tkv; c0 += KMEAN_CHUNK) {
                int c1 = std::min(Tkv, c0 + KMEAN_CHUNK);
                for (int d = 0; d < D; ++d) {
                    double part = 0.0;
                    for (int t = c0; t < c1; ++t)
                        part += (double)bf16_decode(k[b * k_sb + t * k_st + h * k_sh + d]);
                    total[d] += part;
                }
            }
            float* kmh = km + bh * D;
            for (int d = 0; d < D; ++d) kmh[d] = (float)(total[d] / (double)Tkv);

            // Q: one scale per gq-token group over all channels.
            for (int g = 0; g < nq; ++g) {
                int t0 = g * gq, t1 = std::min(Tq, t0 + gq);
                float amax = 0.0f;
                for (int t = t0; t < t1; ++t)
                    for (int d = 0; d < D; ++d)
                        amax = std::max(amax, std::fabs(bf16_decode(q[b * q_sb + t * q_st + h * q_sh + d])));
                float s = amax / 127.0f;
                float inv = amax > 0.0f ? 127.0f / amax : 0.0f;
                sq[bh * nq + g] = s;
                for (int t = t0; t < t1; ++t)
                    for (int d = 0; d < D; ++d) {
                        float x = bf16_decode(q[b * q_sb + t * q_st + h * q_sh + d]);
                        q8[(bh * Tq + t) * D + d] = amax > 0.0f ? quant_i8(x, inv) : 0;
                    }
            }
            // K: smooth, then one scale per gk-token group.
            for (int g = 0; g < nk; ++g) {
                int t0 = g * gk, t1 = std::min(Tkv, t0 + gk);
                float amax = 0.0f;
                for (int t = t0; t < t1; ++t)
                    for (int d = 0; d < D; ++d) {
                        float ks = bf16_decode(k[b * k_sb + t * k_st + h * k_sh + d]) - kmh[d];
                        amax = std::max(amax, std::fabs(ks));
                    }
                float s = amax / 127.0f;
                float inv = amax > 0.0f ? 127.0f / amax : 0.0f;
                sk[bh * nk + g] = s;
                for (int t = t0; t < t1; ++t)
                    for (int d = 0; d < D; ++d) {
                        float ks = bf16_decode(k[b * k_sb + t * k_st + h * k_sh + d]) - kmh[d];
                        k8[(bh * Tkv + t) * D + d] = amax > 0.0f ? quant_i8(ks, inv) : 0;
                    }
            }
            // V: one scale per channel over all valid tokens, FP8 E4M3 words.
            for (int d = 0; d < D; ++d) {
                float amax = 0.0f;
                for (int t = 0; t < Tkv; ++t)
                    amax = std::max(amax, std::fabs(bf16_decode(v[b * v_sb + t * v_st + h * v_sh + d])));
                sv[bh * D + d] = amax / 448.0f;
                float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
                for (int t = 0; t < Tkv; ++t) {
                    float x = bf16_decode(v[b * v_sb + t * v_st + h * v_sh + d]);
                    v8[(bh * Tkv + t) * D + d] = amax > 0.0f ? e4m3_encode(x * inv) : 0;
                }
            }
        }
    return 0;
}

// ------------------------------------------------------ Q/K norm + RoPE ----
// Per-head RMSNorm over the D channels of each (b, t, h) row followed by the
// rotary embedding of channel pairs (2i, 2i+1), the Q/K preparation that the
// pages' H3 block runs before attention ("Norm and RoPE" in the representative
// block table; fused into the attention's input path in Component 2, item 1).
// The pages fix neither formula; the reading taken, step by step:
//   ss  = sum of x_c^2 in FP32 (the precision RMSNorm layers usually accumulate
//         in): the D/8 slices of 8 channels are each summed in channel order,
//         then the slice sums are added pairwise, halving the count each time:
//         slice s += slice s + w for s < w, w = D/16, ..., 2, 1 (for D = 128:
//         s + 8, then s + 4, s + 2, s + 1); every product and sum is rounded
//         separately;
//   ms  = ss / D;  r = 1 / sqrt(ms + eps)   (FP32, each step rounded);
//   n_c = bf16(x_c * r);  z_c = bf16(n_c * gamma_c)   (the norm output, BF16);
//   out_2i   = bf16(z_2i * cos_i - z_2i+1 * sin_i)   (FP32, each product and the
//   out_2i+1 = bf16(z_2i+1 * cos_i + z_2i * sin_i)    sum rounded; no FMA).
// x is [B, T, H, D] BF16 with element strides (sb, st, sh); cos, sin are
// [T, D/2] FP32 (row t = token t); out is dense [B, T, H, D] BF16.
int orc_qk_norm_rope(const uint16_t* x, int64_t sb, int64_t st, int64_t sh, int B, int T, int H, int D,
                     const float* gamma, float eps, const float* cosv, const float* sinv, uint16_t* out) {
    if (B < 1 || T < 1 || H < 1 || D < 16 || D % 16 != 0 || !(eps > 0.0f)) return -1;
    const int nslice = D / 8;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            std::vector<float> part(nslice);
            std::vector<float> z(D);
            for (int h = 0; h < H; ++h) {
                const uint16_t* xr = x + b * sb + t * st + h * sh;
                for (int s = 0; s < nslice; ++s) {
                    float acc = 0.0f;
                    for (int c = 8 * s; c < 8 * s + 8; ++c) {
                        const float xc = bf16_decode(xr[c]);
                        acc += xc * xc;
                    }
                    part[s] = acc;
                }
                for (int w = nslice / 2; w >= 1; w /= 2)
                    for (int s = 0; s < w; ++s) part[s] += part[s + w];
                const float ms = part[0] / (float)D;
                const float den = std::sqrt(ms + eps);
                const float r = 1.0f / den;
                for (int c = 0; c < D; ++c) {
                    const float n = bf16_decode(bf16_encode(bf16_decode(xr[c]) * r));
                    z[c] = bf16_decode(bf16_encode(n * gamma[c]));
                }
                uint16_t* o = out + (((int64_t)b * T + t) * H + h) * D;
                for (int i = 0; i < D / 2; ++i) {
                    const float cs = cosv[(int64_t)t * (D / 2) + i], sn = sinv[(int64_t)t * (D / 2) + i];
                    const float a = z[2 * i], bb = z[2 * i + 1];
                    o[2 * i] = bf16_encode(a * cs - bb * sn);
                    o[2 * i + 1] = bf16_encode(bb * cs + a * sn);
                }
            }
        }
    return 0;
}

// --------------------------------------------------------------- scores -----
// Exact INT32 QK^T for rows [i0, i0+ni) and keys [j0, j0+nj) of head (b, h):
// out[(i-i0)*nj + (j-j0)] = sum_d q8[i,d] * k8[j,d].
int orc_scores(const int8_t* q8, const int8_t* k8, int B, int Tq, int Tkv, int H, int D,
               int b, int h, int i0, int ni, int j0, int nj, int32_t* out) {
    if (b < 0 || b >= B || h < 0 || h >= H || i0 < 0 || j0 < 0 || i0 + ni > Tq || j0 + nj > Tkv) return -1;
    const int64_t bh = (int64_t)b * H + h;
    for (int i = 0; i < ni; ++i)
        for (int j = 0; j < nj; ++j) {
            const int8_t* qr = q8 + (bh * Tq + i0 + i) * D;
            const int8_t* kr = k8 + (bh * Tkv + j0 + j) * D;
            int32_t acc = 0;
            for (int d = 0; d < D; ++d) acc += (int32_t)qr[d] * (int32_t)kr[d];
            out[(int64_t)i * nj + j] = acc;
        }
    return 0;
}

// ------------------------------------------------------------- attention ----
// One query row (b, h, i) through the online-softmax policy.  Optional traces
// (any pointer may be null):
//   acc_tr[Tkv] int32 scores, t_tr[Tkv] f32 log2-domain scores,
//   p8_tr[Tkv] probability words, m_tr/d_tr/alpha_tr[n_epochs] per epoch,
//   ro_tr[D] final RO, r_tr[1] final reciprocal.
static void attend_row(const int8_t* q8, const int8_t* k8, const uint8_t* v8,
                       const float* sq, const float* sk, const float* sv,
                       int Tq, int Tkv, int H, int D, int gq, int gk, float c, int epoch,
                       int b, int h, int i, uint16_t* out_row,
                       int32_t* acc_tr, float* t_tr, uint8_t* p8_tr,
                       float* m_tr, float* d_tr, float* alpha_tr, float* ro_tr, float* r_tr) {
    const int64_t bh = (int64_t)b * H + h;
    const int nq = (Tq + gq - 1) / gq, nk = (Tkv + gk - 1) / gk;
    const int8_t* qr = q8 + (bh * Tq + i) * D;
    const float sqi = sq[bh * nq + i / gq];
    std::vector<float> ro(D, 0.0f), pv(D), t(epoch), p(epoch);
    std::vector<uint8_t> p8(epoch);
    float m = -std::numeric_limits<float>::infinity();
    float dsum = 0.0f;
    int e = 0;
    for (int j0 = 0; j0 < Tkv; j0 += epoch, ++e) {
        const int n = std::min(epoch, Tkv - j0);
        // INT8 QK^T, exact INT32; dequantize into the log2 domain.
        float mloc = -std::numeric_limits<float>::infinity();
        for (int jj = 0; jj < n; ++jj) {
            const int j = j0 + jj;
            const int8_t* kr = k8 + (bh * Tkv + j) * D;
            int32_t acc = 0;
            for (int d = 0; d < D; ++d) acc += (int32_t)qr[d] * (int32_t)kr[d];
            const float f = (sqi * sk[bh * nk + j / gk]) * c;
            t[jj] = (float)acc * f;
            if (acc_tr) acc_tr[j] = acc;
            if (t_tr) t_tr[j] = t[jj];
            mloc = std::max(mloc, t[jj]);
        }
        // Online softmax update.
        const float m_new = std::max(m, mloc);
        const float alpha = std::isinf(m) && m < 0 ? 0.0f : std::exp2(m - m_new);
        float esum = 0.0f;
        for (int jj = 0; jj < n; ++jj) {
            p[jj] = std::exp2(t[jj] - m_new);
            esum += p[jj];
            p8[jj] = e4m3_encode(448.0f * p[jj]);
            if (p8_tr) p8_tr[j0 + jj] = p8[jj];
        }
        dsum = dsum * alpha + esum;
        // FP8 P times FP8 V, FP32 sums in ascending key order.
        const float* dec = e4m3_table().v;
        for (int cc = 0; cc < D; ++cc) pv[cc] = 0.0f;
        for (int jj = 0; jj < n; ++jj) {
            const float pj = dec[p8[jj]];
            const uint8_t* vr = v8 + (bh * Tkv + j0 + jj) * D;
            for (int cc = 0; cc < D; ++cc) pv[cc] += pj * dec[vr[cc]];
        }
        for (int cc = 0; cc < D; ++cc) ro[cc] = ro[cc] * alpha + pv[cc];
        m = m_new;
        if (m_tr) m_tr[e] = m;
        if (d_tr) d_tr[e] = dsum;
        if (alpha_tr) alpha_tr[e] = alpha;
    }
    const float r = 1.0f / dsum;
    if (r_tr) *r_tr = r;
    for (int cc = 0; cc < D; ++cc) {
        if (ro_tr) ro_tr[cc] = ro[cc];
        const float svs = sv[bh * D + cc] / 448.0f;
        out_row[cc] = bf16_encode((ro[cc] * r) * svs);
    }
}

// Output rows for a list of (b, h, i) triples; out is [n_rows, D] BF16 bits.
// m_out / d_out (optional) receive the final running max and sum per row.
int orc_attend_rows(const int8_t* q8, const int8_t* k8, const uint8_t* v8,
                    const float* sq, const float* sk, const float* sv,
                    int B, int Tq, int Tkv, int H, int D, int gq, int gk,
                    float scale, int epoch, int n_rows, const int32_t* rows,
                    uint16_t* out, float* m_out, float* d_out) {
    if (B < 1 || Tq < 1 || Tkv < 1 || H < 1 || D < 1 || epoch < 1) return -1;
    for (int r = 0; r < n_rows; ++r) {
        int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= Tq) return -1;
    }
    const float c = orc_log2_scale(scale);
    const int n_epochs = (Tkv + epoch - 1) / epoch;
#pragma omp parallel
    {
        std::vector<float> mtr(n_epochs), dtr(n_epochs);
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < n_rows; ++r) {
            int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            attend_row(q8, k8, v8, sq, sk, sv, Tq, Tkv, H, D, gq, gk, c, epoch, b, h, i,
                       out + (int64_t)r * D, nullptr, nullptr, nullptr,
                       mtr.data(), dtr.data(), nullptr, nullptr, nullptr);
            if (m_out) m_out[r] = mtr[n_epochs - 1];
            if (d_out) d_out[r] = dtr[n_epochs - 1];
        }
    }
    return 0;
}

// Full checkpoint trace of one row (see attend_row for the buffers).
int orc_row_trace(const int8_t* q8, const int8_t* k8, const uint8_t* v8,
                  const float* sq, const float* sk, const float* sv,
                  int B, int Tq, int Tkv, int H, int D, int gq, int gk,
                  float scale, int epoch, int b, int h, int i, uint16_t* out_row,
                  int32_t* acc_tr, float* t_tr, uint8_t* p8_tr,
                  float* m_tr, float* d_tr, float* alpha_tr, float* ro_tr, float* r_tr) {
    if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= Tq || epoch < 1) return -1;
    attend_row(q8, k8, v8, sq, sk, sv, Tq, Tkv, H, D, gq, gk, orc_log2_scale(scale), epoch, b, h, i,
               out_row, acc_tr, t_tr, p8_tr, m_tr, d_tr, alpha_tr, ro_tr, r_tr);
    return 0;
}

}  // extern "C"
