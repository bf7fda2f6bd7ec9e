// Host oracle for group-wise affine quantization and the quantized products.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, plain CPU statement of what
// the CUDA library computes. Only the tests, the smoke check and the bench's
// CPU-baseline leg load it. It shares no code, header, table or helper with the
// CUDA library, and the CUDA library never calls it.
//
// Sources (nuvec documentation pages):
//   [Q-Affine]   "Docs / Quantization", section "Affine": a row is cut into
//                runs of group_size values; each run carries a scale and a
//                bias; every value is stored as a small unsigned integer, many
//                to a 32-bit word; w is approximately scale * code + bias;
//                4-bit codes with 64-value groups cost roughly 4.5 bits each.
//   [Q-Example]  same section, the example: quantize W [out, in], then
//                quantized_matmul(q, transpose=true) is x . w^T.
//   [Q-Products] "Docs / Quantization", section "Products on the GPU".
//   [Q-MoE]      "Docs / Quantization", section "Mixture of experts":
//                in gather_qmm every row meets the weights of its own expert.
//   [Crate-Quantized] nuvec crate docs, "Structs": Quantized holds uint32
//                codes, one scale per group in the weights' dtype, biases.
//
// What the pages leave open, and the reading taken here (all listed in the
// design notes):
//   * quantizer arithmetic: scale = (max - min) / (2^bits - 1), bias = min,
//     code = clamp(round((w - bias) / scale), 0, 2^bits - 1), every step an
//     IEEE fp32 operation (subtract, divide) rounded to nearest-even;
//   * round() is round-half-to-even (the IEEE default mode);
//   * the codes use the unrounded fp32 scale and bias; the stored scale and
//     bias are then cast to the weights' dtype (bf16: round-to-nearest-even);
//   * a constant group (scale == 0) gets code 0 everywhere;
//   * a group holding both -0 and +0 has minimum -0 and maximum +0;
//   * code j of a uint32 word sits at bits [j*bits, (j+1)*bits);
//   * the product's reference value is the fp64 dot of x with the dequantized
//     weights (stored scale and bias), summed in k order.
//
// Pins: every function here is checked in tests/test_oracle_pins.py against
// closed forms and brute force (hand-built integer groups, pack words written
// out from the bit definition, exact integer products, the round-trip bound).
//
// Build: g++ -O2 -ffp-contract=off -fopenmp -fPIC -shared (no fast-math): fp32
// arithmetic on x86-64 is SSE, so each float operation rounds once, as IEEE
// specifies. Output elements are computed independently and each sum runs in
// k order, so results do not depend on the thread count.

#include <cstdint>
#include <cstring>
#include <cmath>
#include <cfenv>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum { DT_F32 = 0, DT_BF16 = 1 };

// ---- storage dtypes ------------------------------------------------------

// bf16 is the upper half of an fp32 bit pattern: widening is exact.
double load_value(const void* base, int dtype, int64_t i) {
    if (dtype == DT_F32) return (double)((const float*)base)[i];
    uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    std::memcpy(&f, &bits, 4);
    return (double)f;
}

float load_f32(const void* base, int dtype, int64_t i) {
    return (float)load_value(base, dtype, i);
}

// Narrow fp32 to bf16 by rounding the fp32 bit pattern to nearest, ties to
// even, at bit 16 (plain integer rounding on the bits; finite inputs).
uint16_t f32_to_bf16(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    uint32_t keep = u >> 16;
    uint32_t rest = u & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1;
    return (uint16_t)keep;
}

void store_value(void* base, int dtype, int64_t i, float v) {
    if (dtype == DT_F32) ((float*)base)[i] = v;
    else ((uint16_t*)base)[i] = f32_to_bf16(v);
}

// ---- packing [Q-Affine]: code j of a word at bits [j*bits, (j+1)*bits) ----

int64_t words_per_row(int64_t cols, int bits) { return cols * bits / 32; }

uint32_t code_at(const uint32_t* codes, int64_t row, int64_t col, int64_t cols, int bits) {
    const int per_word = 32 / bits;
    uint32_t word = codes[row * words_per_row(cols, bits) + col / per_word];
    int j = (int)(col % per_word);
    return (word >> (j * bits)) & ((1u << bits) - 1u);
}

// ---- dequantize [Q-Affine]: w_hat = scale * code + bias, in fp64 ----------

double dequant_at(const uint32_t* codes, const void* scales, const void* biases, int sdtype,
                  int64_t row, int64_t col, int64_t cols, int gs, int bits) {
    int64_t g = row * (cols / gs) + col / gs;
    double s = load_value(scales, sdtype, g);
    double b = load_value(biases, sdtype, g);
    return s * (double)code_at(codes, row, col, cols, bits) + b;
}

// ---- the stored dequantized value [Q-Affine, Crate-Quantized] --------------
// The dequantized weight, as the dequantizer stores it, is the exact value
// scale * code + bias rounded once (to nearest, ties to even) to the scales'
// dtype. Steps:
//   1. p = scale * code is exact in fp64 (at most 24 + 8 significant bits);
//   2. p + bias = sum + err exactly (the two-sum of Knuth), sum rounded;
//   3. the round-to-odd value of the exact sum at fp64 precision: sum itself
//      when err == 0, else whichever of sum and its neighbour towards err has
//      an odd last bit;
//   4. that value rounded to nearest even at the dtype's precision. A
//      rounding to odd at 53 bits followed by a rounding to at most 51 bits
//      equals a single rounding of the exact value (the odd bit records that
//      the exact value lies strictly between the two 53-bit neighbours).
double round_to_odd_sum(double p, double b) {
    const double sum = p + b;
    const double bb = sum - p;
    const double err = (p - (sum - bb)) + (b - bb);
    if (err == 0.0 || !std::isfinite(sum)) return sum;
    uint64_t u;
    std::memcpy(&u, &sum, 8);
    if (u & 1u) return sum;
    return std::nextafter(sum, err > 0.0 ? INFINITY : -INFINITY);
}

// fp64 -> bf16 bit pattern, round to nearest even at 8 significant bits
// (quantum 2^-133 below the smallest normal 2^-126), infinity past the largest
// finite value. Written from the format: 1 sign, 8 exponent, 7 fraction bits.
uint16_t f64_to_bf16(double d) {
    const uint16_t sign = std::signbit(d) ? 0x8000u : 0u;
    const double a = std::fabs(d);
    if (a == 0.0) return sign;
    if (!std::isfinite(a)) return (uint16_t)(sign | 0x7F80u);
    int e = 0;
    std::frexp(a, &e);                  // a = m * 2^e, m in [0.5, 1)
    int q = e - 8;                      // exponent of the last kept bit
    if (q < -133) q = -133;
    const double r = std::ldexp(std::nearbyint(std::ldexp(a, -q)), q);  // ties to even
    if (r >= 0x1p128) return (uint16_t)(sign | 0x7F80u);
    const float f = (float)r;           // exact: r has at most 8 significant bits
    uint32_t bits;
    std::memcpy(&bits, &f, 4);
    return (uint16_t)(sign | (bits >> 16));
}

// fp64 -> fp32, round to nearest even (the conversion of the default mode),
// infinity past the largest finite value.
float f64_to_f32(double d) {
    if (std::isfinite(d) && std::fabs(d) >= 0x1p128) return std::signbit(d) ? -INFINITY : INFINITY;
    return (float)d;
}

bool valid_quant(int64_t cols, int gs, int bits) {
    if (gs != 32 && gs != 64 && gs != 128) return false;
    if (bits != 1 && bits != 2 && bits != 4 && bits != 8) return false;
    return cols > 0 && cols % gs == 0;
}

// One output element of a product: sum_k x[k] * w_hat(k), sequential in k.
// transpose = 1: the weights are stored [N, K] (row n holds output n).
// transpose = 0: the weights are stored [K, N] (row k), grouped along N.
void dot_one(const void* x_row, int xdtype, int64_t K, int64_t N, int64_t n,
             const uint32_t* codes, const void* scales, const void* biases, int sdtype,
             int gs, int bits, int transpose, double* y, double* a) {
    double acc = 0.0, mag = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double xv = load_value(x_row, xdtype, k);
        double wv = transpose ? dequant_at(codes, scales, biases, sdtype, n, k, K, gs, bits)
                              : dequant_at(codes, scales, biases, sdtype, k, n, N, gs, bits);
        double p = xv * wv;
        acc += p;
        mag += std::fabs(p);
    }
    *y = acc;
    *a = mag;
}

const void* row_ptr(const void* base, int dtype, int64_t row, int64_t len) {
    size_t esz = dtype == DT_F32 ? 4 : 2;
    return (const char*)base + (size_t)row * (size_t)len * esz;
}

// ---- floating-point modes ["Docs / Quantization", section "Floating-point
// formats": every value a small float, one shared scale per group stored as
// a uint8 code, no biases; dequantized to bfloat16]. The pages' table of the
// formats did not survive extraction, so the formats are the published
// definitions of the three names:
//   MXFP4: E2M1 values, one E8M0 scale per 32 values;
//   MXFP8: E4M3 values (no infinities), one E8M0 scale per 32 values;
//   NVFP4: E2M1 values, one E4M3 scale per 16 values.
// Codes pack like the affine codes (code j of a word at bits [j*b, (j+1)*b)).
enum { FP_MXFP4 = 1, FP_MXFP8 = 2, FP_NVFP4 = 3 };

int fp_group(int mode) { return mode == FP_NVFP4 ? 16 : 32; }
int fp_bits(int mode) { return mode == FP_MXFP8 ? 8 : 4; }

// E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0; exponent 0
// is subnormal (0.5 * mantissa).
double e2m1_value(uint32_t c) {
    const int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    const double mag = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}
// E4M3 without infinities: sign bit 7, exponent bits 6..3 (bias 7), mantissa
// bits 2..0; exponent 0 is subnormal (mantissa / 8 * 2^-6); S.1111.111 is NaN.
double e4m3_value(uint32_t c) {
    const int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return std::nan("");
    const double mag = e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}
// E8M0: 2^(code - 127); code 255 is NaN.
double e8m0_value(uint32_t c) { return c == 255 ? std::nan("") : std::ldexp(1.0, (int)c - 127); }

// The code of a finite value in E2M1 (elem = 0) or E4M3 (elem = 1): the sign
// of v, and the magnitude of the grid nearest to |v|, ties to the code whose
// mantissa field is even, magnitudes past the largest finite one saturated to
// it. Brute force over the grid.
uint32_t nearest_code(double v, int elem) {
    const uint32_t sign_bit = elem == 0 ? 8u : 128u;
    const uint32_t top = elem == 0 ? 7u : 126u;  // largest finite magnitude code
    const double a = std::fabs(v);
    uint32_t best = 0;
    double best_d = a;  // distance to code 0 (zero)
    for (uint32_t c = 1; c <= top; ++c) {
        const double g = elem == 0 ? e2m1_value(c) : e4m3_value(c);
        const double d = std::fabs(a - g);
        if (d < best_d || (d == best_d && (c & 1u) == 0u)) { best = c; best_d = d; }
    }
    const double gmax = elem == 0 ? e2m1_value(top) : e4m3_value(top);
    if (a >= gmax) best = top;
    return std::signbit(v) ? (best | sign_bit) : best;
}

// Value of element code c and scale code s of a mode.
double fp_element(int mode, uint32_t c) { return mode == FP_MXFP8 ? e4m3_value(c) : e2m1_value(c); }
double fp_scale(int mode, uint32_t s) { return mode == FP_NVFP4 ? e4m3_value(s) : e8m0_value(s); }

double fp_dequant_at(const uint32_t* codes, const uint8_t* scales, int mode, int64_t row, int64_t col,
                     int64_t cols) {
    const int gs = fp_group(mode), bits = fp_bits(mode);
    const uint32_t c = code_at(codes, row, col, cols, bits);
    return fp_element(mode, c) * fp_scale(mode, scales[row * (cols / gs) + col / gs]);
}

}  // namespace

extern "C" {

int orc_threads() {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

// fp32 -> bf16 bit patterns, round to nearest even.
void orc_cast_bf16(const float* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16(in[i]);
}

// Affine quantizer [Q-Affine, Q-Example, Crate-Quantized].
// w [rows, cols] in `dtype` (0 = fp32, 1 = bf16), grouped along cols.
// Writes codes [rows, cols*bits/32] uint32 and scales/biases
// [rows, cols/group_size] in `dtype`. Returns 0, or -1 on bad arguments.
int orc_quantize_affine(const void* w, int dtype, int64_t rows, int64_t cols, int gs,
                        int bits, uint32_t* codes, void* scales, void* biases) {
    if (!valid_quant(cols, gs, bits) || rows < 0) return -1;
    if (std::fegetround() != FE_TONEAREST) return -1;
    const int64_t groups = cols / gs;
    const int per_word = 32 / bits;
    const float levels = (float)((1u << bits) - 1u);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < groups; ++g) {
            const int64_t c0 = g * gs;
            // Step 1: the group's minimum and maximum.
            float mn = load_f32(w, dtype, r * cols + c0), mx = mn;
            // A group holding both zeros has minimum -0 and maximum +0, so the
            // result does not depend on the order the values are visited in.
            for (int i = 1; i < gs; ++i) {
                float v = load_f32(w, dtype, r * cols + c0 + i);
                if (v < mn || (v == mn && std::signbit(v))) mn = v;
                if (v > mx || (v == mx && !std::signbit(v))) mx = v;
            }
            // Step 2: scale spreads the range over the 2^bits - 1 steps; bias = min.
            float range = mx - mn;
            float scale = range / levels;
            float bias = mn;
            // Step 3: one code per value, round-half-even, clamped.
            for (int i = 0; i < gs; ++i) {
                uint32_t q = 0;
                if (scale != 0.0f) {
                    float v = load_f32(w, dtype, r * cols + c0 + i);
                    float t = (v - bias) / scale;
                    float rq = std::nearbyint(t);
                    if (rq < 0.0f) rq = 0.0f;
                    if (rq > levels) rq = levels;
                    q = (uint32_t)rq;
                }
                // Step 4: pack code (c0 + i) into its word.
                int64_t col = c0 + i;
                int64_t wi = r * words_per_row(cols, bits) + col / per_word;
                int j = (int)(col % per_word);
                if (j == 0) codes[wi] = 0u;
                codes[wi] |= q << (j * bits);
            }
            // Step 5: store scale and bias in the weights' dtype.
            store_value(scales, dtype, r * groups + g, scale);
            store_value(biases, dtype, r * groups + g, bias);
        }
    }
    return 0;
}

// Dequantize to fp64: out[r, c] = scale * code + bias [Q-Affine].
int orc_dequantize(const uint32_t* codes, const void* scales, const void* biases, int sdtype,
                   int64_t rows, int64_t cols, int gs, int bits, double* out) {
    if (!valid_quant(cols, gs, bits)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = dequant_at(codes, scales, biases, sdtype, r, c, cols, gs, bits);
    return 0;
}

// The dequantized weights as stored: out[r, c] = scale * code + bias rounded
// once to the scales' dtype (see round_to_odd_sum) [Q-Affine, Crate-Quantized].
int orc_dequantize_stored(const uint32_t* codes, const void* scales, const void* biases,
                          int sdtype, int64_t rows, int64_t cols, int gs, int bits, void* out) {
    if (!valid_quant(cols, gs, bits)) return -1;
    if (std::fegetround() != FE_TONEAREST) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            const int64_t g = r * (cols / gs) + c / gs;
            const double p = load_value(scales, sdtype, g) * (double)code_at(codes, r, c, cols, bits);
            const double v = round_to_odd_sum(p, load_value(biases, sdtype, g));
            if (sdtype == DT_F32) ((float*)out)[r * cols + c] = f64_to_f32(v);
            else ((uint16_t*)out)[r * cols + c] = f64_to_bf16(v);
        }
    return 0;
}

// Quantized product [Q-Example, Q-Products]: y[m, n] = sum_k x[m, k] * w_hat(n, k)
// with transpose = 1 (weights [N, K]); transpose = 0 uses weights [K, N].
// Also returns a[m, n] = sum_k |x[m, k] * w_hat|, the scale of the tolerance.
int orc_qmm(const void* x, int xdtype, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
            const void* scales, const void* biases, int sdtype, int gs, int bits, int transpose,
            double* y, double* a) {
    if (!valid_quant(transpose ? K : N, gs, bits)) return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            dot_one(row_ptr(x, xdtype, m, K), xdtype, K, N, n, codes, scales, biases, sdtype,
                    gs, bits, transpose, &y[m * N + n], &a[m * N + n]);
    return 0;
}

// The same product at S chosen output positions (m_idx[s], n_idx[s]) only.
int orc_qmm_sampled(const void* x, int xdtype, int64_t M, int64_t K, int64_t N,
                    const uint32_t* codes, const void* scales, const void* biases, int sdtype,
                    int gs, int bits, int transpose, int64_t S, const int64_t* m_idx,
                    const int64_t* n_idx, double* y, double* a) {
    if (!valid_quant(transpose ? K : N, gs, bits)) return -1;
    for (int64_t s = 0; s < S; ++s)
        if (m_idx[s] < 0 || m_idx[s] >= M || n_idx[s] < 0 || n_idx[s] >= N) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < S; ++s)
        dot_one(row_ptr(x, xdtype, m_idx[s], K), xdtype, K, N, n_idx[s], codes, scales, biases,
                sdtype, gs, bits, transpose, &y[s], &a[s]);
    return 0;
}

// Mixture-of-experts product [Q-MoE]: for each pair r, output row r is
// x[lhs[r]] times expert rhs[r]'s weights (experts stored [E, N, K] with
// transpose = 1, or [E, K, N] with transpose = 0). lhs may be null (identity).
// Returns -1 if an index is out of range.
int orc_gather_qmm(const void* x, int xdtype, int64_t x_rows, int64_t K, const uint32_t* lhs,
                   const uint32_t* rhs, int64_t R, int64_t E, int64_t N, const uint32_t* codes,
                   const void* scales, const void* biases, int sdtype, int gs, int bits,
                   int transpose, double* y, double* a) {
    if (!valid_quant(transpose ? K : N, gs, bits)) return -1;
    for (int64_t r = 0; r < R; ++r) {
        int64_t t = lhs ? (int64_t)lhs[r] : r;
        if (t >= x_rows || (int64_t)rhs[r] >= E) return -1;
    }
    const int64_t words_e = N * K * bits / 32;
    const int64_t groups_e = N * K / gs;
    const size_t sz = sdtype == DT_F32 ? 4 : 2;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t n = 0; n < N; ++n) {
            int64_t t = lhs ? (int64_t)lhs[r] : r;
            int64_t e = (int64_t)rhs[r];
            dot_one(row_ptr(x, xdtype, t, K), xdtype, K, N, n, codes + e * words_e,
                    (const char*)scales + (size_t)(e * groups_e) * sz,
                    (const char*)biases + (size_t)(e * groups_e) * sz, sdtype, gs, bits,
                    transpose, &y[r * N + n], &a[r * N + n]);
        }
    return 0;
}

// The same gather at S chosen (pair, output) positions.
int orc_gather_qmm_sampled(const void* x, int xdtype, int64_t x_rows, int64_t K,
                           const uint32_t* lhs, const uint32_t* rhs, int64_t R, int64_t E,
                           int64_t N, const uint32_t* codes, const void* scales,
                           const void* biases, int sdtype, int gs, int bits, int transpose,
                           int64_t S, const int64_t* r_idx, const int64_t* n_idx, double* y,
                           double* a) {
    if (!valid_quant(transpose ? K : N, gs, bits)) return -1;
    for (int64_t s = 0; s < S; ++s) {
        int64_t r = r_idx[s];
        if (r < 0 || r >= R || n_idx[s] < 0 || n_idx[s] >= N) return -1;
        int64_t t = lhs ? (int64_t)lhs[r] : r;
        if (t >= x_rows || (int64_t)rhs[r] >= E) return -1;
    }
    const int64_t words_e = N * K * bits / 32;
    const int64_t groups_e = N * K / gs;
    const size_t sz = sdtype == DT_F32 ? 4 : 2;
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < S; ++s) {
        int64_t r = r_idx[s];
        int64_t t = lhs ? (int64_t)lhs[r] : r;
        int64_t e = (int64_t)rhs[r];
        dot_one(row_ptr(x, xdtype, t, K), xdtype, K, N, n_idx[s], codes + e * words_e,
                (const char*)scales + (size_t)(e * groups_e) * sz,
                (const char*)biases + (size_t)(e * groups_e) * sz, sdtype, gs, bits, transpose,
                &y[s], &a[s]);
    }
    return 0;
}

// Gather with full-precision experts [Q-MoE: every row meets the weights of
// its own expert; crate docs: gather_mm beside gather_qmm]:
// y[r, n] = sum_k x[lhs[r], k] * w[rhs[r], n, k], w [E, N, K] in `wdtype`,
// fp64, sequential in k; a[r, n] = sum_k |x * w|. Returns -1 if an index is
// out of range.
int orc_gather_mm(const void* x, int xdtype, int64_t x_rows, int64_t K, const uint32_t* lhs,
                  const uint32_t* rhs, int64_t R, int64_t E, int64_t N, const void* w,
                  int wdtype, double* y, double* a) {
    for (int64_t r = 0; r < R; ++r) {
        int64_t t = lhs ? (int64_t)lhs[r] : r;
        if (t >= x_rows || (int64_t)rhs[r] >= E) return -1;
    }
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t n = 0; n < N; ++n) {
            const int64_t t = lhs ? (int64_t)lhs[r] : r;
            const int64_t wrow = ((int64_t)rhs[r] * N + n) * K;
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = load_value(x, xdtype, t * K + k) * load_value(w, wdtype, wrow + k);
                acc += p;
                mag += std::fabs(p);
            }
            y[r * N + n] = acc;
            a[r * N + n] = mag;
        }
    return 0;
}

// Mixture-of-experts block with a SwiGLU expert [Q-MoE; the routed pass of
// gate, up and down products], every product through quantized weights:
//   for token t and each of its top-k (expert e = ids[t, j], weight rw[t, j]):
//     g_i = sum_k x[t, k] * wg_hat[e, i, k],  u_i = sum_k x[t, k] * wu_hat[e, i, k]
//     h_i = silu(g_i) * u_i,  silu(z) = z / (1 + exp(-z))
//     y[t, n] += rw[t, j] * sum_i h_i * wd_hat[e, n, i]
// Gate and up weights are [E, I, K] grouped along K, down weights [E, K, I]
// grouped along I; all share one group size, width and scale dtype. fp64
// throughout, sums in index order. Out-of-range expert ids are skipped (they
// contribute nothing), so a caller can state them.
// a[t, n] is the scale of the block's tolerance: the product tolerance
// carried to first order through h = silu(g) * u, each term doubled for the
// rounding of the intermediate g and h to the activations' dtype:
//   a[t, n] = sum_j |rw| sum_i |wd_hat[e, n, i]| *
//             2 (|h_i| + |silu'(g_i) u_i| a_g,i + |silu(g_i)| a_u,i),
// with a_g,i = sum_k |x_k wg_hat[e, i, k]|, a_u,i likewise, and
// silu'(z) = s(z) (1 + z (1 - s(z))), s(z) = 1 / (1 + exp(-z)).
// Returns -1 on a bad quantization.
int orc_moe_swiglu(const void* x, int xdtype, int64_t T, int64_t K, const uint32_t* ids,
                   const float* rw, int topk, int64_t E, int64_t I,
                   const uint32_t* g_codes, const void* g_scales, const void* g_biases,
                   const uint32_t* u_codes, const void* u_scales, const void* u_biases,
                   const uint32_t* d_codes, const void* d_scales, const void* d_biases,
                   int sdtype, int gs, int bits, double* y, double* a) {
    if (!valid_quant(K, gs, bits) || !valid_quant(I, gs, bits) || topk < 1) return -1;
    const size_t sz = sdtype == DT_F32 ? 4 : 2;
    const int64_t gu_words = I * K * bits / 32, gu_groups = I * K / gs;   // per expert
    const int64_t d_words = K * I * bits / 32, d_groups = K * I / gs;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* yt = y + t * K;
        double* at = a + t * K;
        for (int64_t n = 0; n < K; ++n) { yt[n] = 0.0; at[n] = 0.0; }
        double* h = new double[I];
        double* eh = new double[I];  // error scale of h_i
        for (int j = 0; j < topk; ++j) {
            const int64_t e = (int64_t)ids[t * topk + j];
            if (e >= E) continue;
            const double w = (double)rw[t * topk + j];
            const uint32_t* gc = g_codes + e * gu_words;
            const uint32_t* uc = u_codes + e * gu_words;
            const char* gsc = (const char*)g_scales + (size_t)(e * gu_groups) * sz;
            const char* gbi = (const char*)g_biases + (size_t)(e * gu_groups) * sz;
            const char* usc = (const char*)u_scales + (size_t)(e * gu_groups) * sz;
            const char* ubi = (const char*)u_biases + (size_t)(e * gu_groups) * sz;
            for (int64_t i = 0; i < I; ++i) {
                double g = 0.0, u = 0.0, ag = 0.0, au = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    const double xv = load_value(x, xdtype, t * K + k);
                    const double pg = xv * dequant_at(gc, gsc, gbi, sdtype, i, k, K, gs, bits);
                    const double pu = xv * dequant_at(uc, usc, ubi, sdtype, i, k, K, gs, bits);
                    g += pg;
                    u += pu;
                    ag += std::fabs(pg);
                    au += std::fabs(pu);
                }
                h[i] = g / (1.0 + std::exp(-g)) * u;
                const double sg = 1.0 / (1.0 + std::exp(-g));
                const double dsilu = sg * (1.0 + g * (1.0 - sg));
                eh[i] = 2.0 * (std::fabs(h[i]) + std::fabs(dsilu * u) * ag + std::fabs(g * sg) * au);
            }
            const uint32_t* dc = d_codes + e * d_words;
            const char* dsc = (const char*)d_scales + (size_t)(e * d_groups) * sz;
            const char* dbi = (const char*)d_biases + (size_t)(e * d_groups) * sz;
            for (int64_t n = 0; n < K; ++n) {
                double acc = 0.0, mag = 0.0;
                for (int64_t i = 0; i < I; ++i) {
                    const double wd = dequant_at(dc, dsc, dbi, sdtype, n, i, I, gs, bits);
                    acc += h[i] * wd;
                    mag += std::fabs(wd) * eh[i];
                }
                yt[n] += w * acc;
                at[n] += std::fabs(w) * mag;
            }
        }
        delete[] h;
        delete[] eh;
    }
    return 0;
}


// Quantizer of the floating-point modes ["Docs / Quantization", section
// "Floating-point formats"; the scale rule is the shared-exponent rule of the
// published microscaling formats, written out step by step]. w [rows, cols]
// in `dtype` (fp32 or bf16), groups along cols. Writes codes [rows,
// cols*bits/32] and scale codes [rows, cols/gs] (uint8). Returns 0, or -1 on
// bad arguments.
//   MXFP4 / MXFP8: amax = max |w| of the group; X = 2^(floor(log2 amax) -
//   emax), emax = 2 (E2M1) or 8 (E4M3), the scale code clamped to 0..254 (an
//   all-zero group gets code 0); each code is the nearest element of w / X
//   (exact: X is a power of two).
//   NVFP4: the scale is fl32(amax / 6) rounded to E4M3; each code is the
//   nearest element of fl32(w / S), S the stored scale (code 0 when S is 0).
int orc_quantize_fp(const void* w, int dtype, int64_t rows, int64_t cols, int mode,
                    uint32_t* codes, uint8_t* scales) {
    if (mode != FP_MXFP4 && mode != FP_MXFP8 && mode != FP_NVFP4) return -1;
    const int gs = fp_group(mode), bits = fp_bits(mode);
    if (rows < 0 || cols <= 0 || cols % gs != 0) return -1;
    if (std::fegetround() != FE_TONEAREST) return -1;
    const int64_t groups = cols / gs;
    const int per_word = 32 / bits;
    const int elem = mode == FP_MXFP8 ? 1 : 0;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < groups; ++g) {
            const int64_t c0 = g * gs;
            // Step 1: the group's largest magnitude.
            float amax = 0.0f;
            for (int i = 0; i < gs; ++i) amax = std::fmax(amax, std::fabs(load_f32(w, dtype, r * cols + c0 + i)));
            // Step 2: the shared scale.
            uint32_t scode = 0;
            if (mode == FP_NVFP4) {
                const float sv = amax / 6.0f;
                scode = nearest_code((double)sv, 1) & 127u;
            } else if (amax > 0.0f) {
                int ex = 0;
                std::frexp((double)amax, &ex);            // amax = f * 2^ex, f in [0.5, 1)
                const int e = (ex - 1) - (elem == 0 ? 2 : 8);  // floor(log2 amax) - emax
                int sc = e + 127;
                if (sc < 0) sc = 0;
                if (sc > 254) sc = 254;
                scode = (uint32_t)sc;
            }
            scales[r * groups + g] = (uint8_t)scode;
            const double sval = fp_scale(mode, scode);
            // Step 3: one element code per value, then pack.
            for (int i = 0; i < gs; ++i) {
                const float v = load_f32(w, dtype, r * cols + c0 + i);
                uint32_t q = 0;
                if (mode == FP_NVFP4) {
                    if (sval != 0.0) q = nearest_code((double)(v / (float)sval), 0);
                } else {
                    q = nearest_code((double)v / sval, elem);
                }
                const int64_t col = c0 + i;
                const int64_t wi = r * words_per_row(cols, bits) + col / per_word;
                const int j = (int)(col % per_word);
                if (j == 0) codes[wi] = 0u;
                codes[wi] |= q << (j * bits);
            }
        }
    }
    return 0;
}

// Dequantized weights of a floating-point mode, element value times scale
// value, as bf16 bit patterns (rounded once to nearest even; exact whenever
// the product is a bf16 number, which it is outside extreme underflow).
int orc_dequantize_fp(const uint32_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                      int mode, uint16_t* out) {
    if (mode != FP_MXFP4 && mode != FP_MXFP8 && mode != FP_NVFP4) return -1;
    if (cols <= 0 || cols % fp_group(mode) != 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = f64_to_bf16(fp_dequant_at(codes, scales, mode, r, c, cols));
    return 0;
}

// Product with floating-point-mode weights [N, K] ("Floating-point formats":
// quantized_matmul(q, transpose = true) in x's dtype): y[m, n] = sum_k
// x[m, k] * w_hat(n, k) in fp64, k in order, and a[m, n] = sum_k |x w_hat|.
int orc_qmm_fp(const void* x, int xdtype, int64_t M, int64_t K, int64_t N, const uint32_t* codes,
               const uint8_t* scales, int mode, double* y, double* a) {
    if (mode != FP_MXFP4 && mode != FP_MXFP8 && mode != FP_NVFP4) return -1;
    if (K <= 0 || K % fp_group(mode) != 0 || M < 0 || N < 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M * N; ++i) {
        const int64_t m = i / N, n = i % N;
        double acc = 0.0, mag = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double p = load_value(x, xdtype, m * K + k) * fp_dequant_at(codes, scales, mode, n, k, K);
            acc += p;
            mag += std::fabs(p);
        }
        y[i] = acc;
        a[i] = mag;
    }
    return 0;
}

// Single values of the formats, for the pins: element (elem 0 = E2M1, 1 =
// E4M3) or scale (2 = E8M0) code -> value, and value -> nearest element code.
double orc_fp_value(int kind, uint32_t code) {
    return kind == 0 ? e2m1_value(code) : kind == 1 ? e4m3_value(code) : e8m0_value(code);
}
uint32_t orc_fp_nearest(int elem, double v) { return nearest_code(v, elem); }

}  // extern "C"
