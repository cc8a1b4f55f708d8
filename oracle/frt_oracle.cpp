// Oracle for the fused non-GEMM layer chain -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, obviously-correct CPU restatement of what the three fused
// ops compute, in fp64, one element at a time, in the order the sources state
// the steps.  It shares no code, header, table or constant with the CUDA
// library; only tests, the smoke check and the bench's CPU-baseline leg may
// load it.  The product path never calls it.
//
// Sources (web pages; cited by title and section):
//   [FR]  "FlashRT kernel fusion: RMSNorm / residual / FP8 / QKV post-processing"
//         (xdnf.cn/news/367260), sections 一..六 and the per-layer table in §二.
//   [FR4] "sm89 prefill FFN megakernel" (FlashRT issue #1), Phase 1/Phase 2 and
//         the correctness paragraph (per-token block-128 FP8 scales, out_scale).
//   [FP]  "Falcon-Perception inference optimisation" (nxmr.cn/news/154322),
//         third technique: interleaved [g0,u0,g1,u1,...] gate/up, relu(g)^2*u,
//         sqrt(2) pre-baked into the gate weights.
//
// Readings taken where the pages are silent are listed in the design notes;
// each function below states the one it relies on.
//
// Parity pins: every exported function is pinned by -m "not gpu" tests
// (closed forms, invariants, library special cases, exhaustive round trips and
// an independent brute-force restatement on tiny inputs).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// Own enumerations (numerically equal to the library's ABI values because
// they are the interface the tests speak, not shared code).
enum { DT_F16 = 0, DT_BF16 = 1 };
enum { Q_STATIC = 0, Q_BLOCK128 = 1 };
enum { ACT_GELU_TANH = 0, ACT_SILU = 1, ACT_RELU2 = 2 };

// ---------------------------------------------------------------- formats --
// IEEE-style binary16 (1/5/10) and bfloat16 (1/8/7) described by their field
// widths; decoding is exact in double.
struct Fmt16 {
  int exp_bits;
  int mant_bits;
};
const Fmt16 kF16 = {5, 10};
const Fmt16 kBF16 = {8, 7};

double decode16(uint16_t b, Fmt16 f) {
  const int bias = (1 << (f.exp_bits - 1)) - 1;
  const int emask = (1 << f.exp_bits) - 1;
  const int sign = (b >> 15) & 1;
  const int e = (b >> f.mant_bits) & emask;
  const int m = b & ((1 << f.mant_bits) - 1);
  double v;
  if (e == 0) {
    v = std::ldexp((double)m, 1 - bias - f.mant_bits);  // subnormal / zero
  } else if (e == emask) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = std::ldexp((double)((1 << f.mant_bits) | m), e - bias - f.mant_bits);
  }
  return sign ? -v : v;
}

// Round the exact real number hi + lo (|lo| at most half an ulp of hi in
// double, as produced by an error-free sum) to the 16-bit format, round to
// nearest, ties to even.  lo only decides exact 16-bit midpoints of hi.
uint16_t round16(double hi, double lo, Fmt16 f) {
  const int bias = (1 << (f.exp_bits - 1)) - 1;
  const int emask = (1 << f.exp_bits) - 1;
  const int emin = 1 - bias, emax = bias;
  const uint16_t sign = std::signbit(hi) ? 0x8000 : 0;
  if (std::isnan(hi)) return (uint16_t)(sign | (emask << f.mant_bits) | (1 << (f.mant_bits - 1)));
  const double a = std::fabs(hi);
  const double l = std::signbit(hi) ? -lo : lo;  // error term, same orientation as a
  if (std::isinf(a)) return (uint16_t)(sign | (emask << f.mant_bits));
  if (a == 0.0) return sign;
  int e2;
  std::frexp(a, &e2);           // a = fr * 2^e2, fr in [0.5, 1)
  int E = e2 - 1;               // floor(log2 a)
  if (E < emin) E = emin;       // subnormal range shares the emin quantum
  const double quantum = std::ldexp(1.0, E - f.mant_bits);
  const double n = a / quantum;  // exact: scaling by a power of two
  const double fl = std::floor(n);
  const double frac = n - fl;
  double m;
  if (frac > 0.5) {
    m = fl + 1.0;
  } else if (frac < 0.5) {
    m = fl;
  } else if (l > 0.0) {
    m = fl + 1.0;               // exact value lies above the midpoint
  } else if (l < 0.0) {
    m = fl;                     // exact value lies below the midpoint
  } else {
    m = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;  // true tie: to even
  }
  if (m == std::ldexp(1.0, f.mant_bits + 1)) {  // carried into the next binade
    E += 1;
    m = std::ldexp(1.0, f.mant_bits);
  }
  if (E > emax) return (uint16_t)(sign | (emask << f.mant_bits));  // overflow: inf
  const uint32_t mi = (uint32_t)m;
  if (mi < (1u << f.mant_bits)) return (uint16_t)(sign | mi);      // subnormal
  return (uint16_t)(sign | ((uint32_t)(E + bias) << f.mant_bits) | (mi - (1u << f.mant_bits)));
}

Fmt16 fmt_of(int dt) { return dt == DT_BF16 ? kBF16 : kF16; }

// Error-free transformation: a + b == s + err exactly (Knuth's TwoSum).
void two_sum(double a, double b, double* s, double* err) {
  const double sum = a + b;
  const double bb = sum - a;
  *err = (a - (sum - bb)) + (b - bb);
  *s = sum;
}

// OCP FP8 E4M3 ("e4m3fn"): bias 7, 3 mantissa bits, no infinities, one NaN
// code per sign (0x7F / 0xFF), largest finite 448, smallest normal 2^-6,
// subnormal step 2^-9.  Round to nearest, ties to even, saturating at +-448.
uint8_t e4m3_encode(double v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t s = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(v);
  if (a >= 448.0) return (uint8_t)(s | 0x7E);
  if (a == 0.0) return s;
  int e2;
  std::frexp(a, &e2);
  int e = e2 - 1;
  if (e < -6) e = -6;
  const double quantum = std::ldexp(1.0, e - 3);
  const double n = a / quantum;
  const double fl = std::floor(n);
  const double frac = n - fl;
  double m;
  if (frac > 0.5) {
    m = fl + 1.0;
  } else if (frac < 0.5) {
    m = fl;
  } else {
    m = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  }
  if (m == 16.0) {
    e += 1;
    m = 8.0;
  }
  const int mi = (int)m;
  if (mi < 8) return (uint8_t)(s | mi);  // subnormal (e == -6)
  return (uint8_t)(s | ((e + 7) << 3) | (mi - 8));
}

double e4m3_decode(uint8_t c) {
  const int sign = c >> 7;
  const int e = (c >> 3) & 0xF;
  const int m = c & 7;
  double v;
  if (e == 0xF && m == 7) {
    v = NAN;
  } else if (e == 0) {
    v = std::ldexp((double)m, -9);
  } else {
    v = std::ldexp((double)(8 + m), e - 7 - 3);
  }
  return sign ? -v : v;
}

// ------------------------------------------------------------ quantisers --
// The FP8 code is an integer decided by floating point, so it is decided in
// one stated precision on both sides: fp32, the precision of the kernels (the
// pages fix none).  The value y (fp64 here) is rounded once to fp32, divided by
// the fp32 scale in fp32 (IEEE, round to nearest), and that quotient is
// encoded.
uint8_t quant_fp32(double y, float s32) {
  const float v = (float)y / s32;
  return e4m3_encode((double)v);
}

// Static per-tensor FP8 ([FR] §六: `_static` = the activation scale is a
// constant).  s is a dequantisation scale (an fp32 value): q = e4m3(y / s),
// y ~ q * s.
void quant_static(const double* y, int64_t n, double s, uint8_t* q) {
  const float s32 = (float)s;
  for (int64_t j = 0; j < n; ++j) q[j] = quant_fp32(y[j], s32);
}

// Per-token block-128 FP8 ([FR4] Phase 2: per-token block-128 quantisation
// with an out_scale per row and block).  Block b covers columns
// [128b, min(128b+128, n)); s_b = amax_b / 448, or 1 when the block is all
// zero; q = e4m3(y / s_b).  `scales` receives the fp64 amax_b / 448; the codes
// use the same scale evaluated in fp32 (fp32(amax_b) / 448 in fp32).
void quant_block128(const double* y, int64_t n, uint8_t* q, double* scales) {
  const int64_t nb = (n + 127) / 128;
  for (int64_t b = 0; b < nb; ++b) {
    const int64_t lo = 128 * b;
    const int64_t hi = (lo + 128 < n) ? lo + 128 : n;
    double amax = 0.0;
    for (int64_t j = lo; j < hi; ++j) amax = std::fmax(amax, std::fabs(y[j]));
    scales[b] = (amax > 0.0) ? amax / 448.0 : 1.0;
    const float s32 = (amax > 0.0) ? (float)amax / 448.0f : 1.0f;
    for (int64_t j = lo; j < hi; ++j) q[j] = quant_fp32(y[j], s32);
  }
}

// ---------------------------------------------------------------- NVFP4 --
// NVFP4 (NEXT-3; the pages' W4A4 path: "residual_add_rms_norm_to_nvfp4",
// "silu_mul_merged_grouped32", NVFP4 producers feeding FP4 GEMMs).  The pages
// name the format only; the reading is NVIDIA's NVFP4:
//   element  e2m1 (1 sign, 2 exponent, 1 mantissa bit): magnitudes
//            0, 0.5, 1, 1.5, 2, 3, 4, 6; round to nearest, ties to even
//            mantissa, saturating at 6; two per byte, element 2j in the low
//            nibble of byte j.
//   block    16 consecutive elements of a row share one unsigned e4m3 scale
//            factor sf; with the per-tensor fp32 global scale gs,
//            y ~ e2m1 * decode(sf) * gs.
//   decision the nearest code to an exact quotient, taken on that quotient
//            rounded once to fp32 (the precision every FP8 decision here is
//            taken in): with y32 the fp32 values and amax32 = max |y32| over
//            the block,
//              sf   = e4m3(fp32(amax32 / (6 gs)))          (RNE, saturating to 448),
//              code = e2m1(fp32(y32 / (decode(sf) gs)))  (RNE, saturating to 6);
//            6 gs and decode(sf) gs are exact in fp64 (at most 28 significant
//            bits), and an fp64 quotient of fp32 operands rounded to fp32 is
//            the correctly rounded fp32 quotient (double rounding is
//            innocuous for division when 53 >= 2 * 24 + 2).  sf == 0 (an
//            all-zero or negligible block) gives all-zero codes.
uint8_t e2m1_encode(double v) {
  const uint8_t s = std::signbit(v) ? 0x8 : 0x0;
  const double a = std::fabs(v);
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  if (!(a < 6.0)) return (uint8_t)(s | 7);  // saturate (NaN inputs are not defined here)
  int best = 0;
  for (int c = 1; c < 8; ++c) {
    const double d = std::fabs(mag[c] - a), db = std::fabs(mag[best] - a);
    if (d < db || (d == db && (c & 1) == 0)) best = c;  // ties to the even mantissa bit
  }
  return (uint8_t)(s | best);
}

double e2m1_decode(uint8_t c) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const double v = mag[c & 7];
  return (c & 0x8) ? -v : v;
}

// One row of n (a multiple of 16) values -> n/2 packed bytes and n/16 scale
// factors (row-major).
void quant_nvfp4_row(const double* y, int64_t n, float gs, uint8_t* packed, uint8_t* sf) {
  const double den = 6.0 * (double)gs;  // exact
  for (int64_t b = 0; b < n / 16; ++b) {
    float y32[16];
    float amax = 0.0f;
    for (int j = 0; j < 16; ++j) {
      y32[j] = (float)y[16 * b + j];
      amax = std::fmax(amax, std::fabs(y32[j]));
    }
    const uint8_t code_sf = e4m3_encode((double)(float)((double)amax / den));
    sf[b] = code_sf;
    const double eff = e4m3_decode(code_sf) * (double)gs;  // exact
    uint8_t q[16];
    for (int j = 0; j < 16; ++j) q[j] = (eff > 0.0) ? e2m1_encode((double)(float)((double)y32[j] / eff)) : 0;
    for (int j = 0; j < 8; ++j) packed[8 * b + j] = (uint8_t)(q[2 * j] | (q[2 * j + 1] << 4));
  }
}

// Byte offset of scale factor (row r, column c) in the 128x4-swizzled layout
// that block-scaled tensor-core GEMMs read: atoms of 128 rows x 4 scale
// columns (512 bytes), atoms laid out row-major over (row / 128, c / 4) with
// ceil(n_cols / 4) atoms per atom-row; inside an atom, row r % 128 = 32 i + k
// and column c % 4 = l sit at byte 16 k + 4 i + l.
int64_t sf_swizzle_offset(int64_t r, int64_t c, int64_t n_cols) {
  const int64_t atoms_per_row = (n_cols + 3) / 4;
  const int64_t atom = (r / 128) * atoms_per_row + c / 4;
  const int64_t rr = r % 128;
  return atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (c % 4);
}

// --------------------------------------------------------------- RMSNorm --
// y_j = h_j * rstd * w_j with rstd = 1 / sqrt(mean(h^2) + eps); w == nullptr
// is the `_noweight` form whose (1 + w) lives in the next GEMM's weights
// ([FR] §三 and the §二.1 naming table).
void rmsnorm(const double* h, int64_t n, const double* w, double eps, double* y) {
  double ss = 0.0;
  for (int64_t j = 0; j < n; ++j) ss += h[j] * h[j];
  const double rstd = 1.0 / std::sqrt(ss / (double)n + eps);
  for (int64_t j = 0; j < n; ++j) y[j] = h[j] * rstd * (w ? w[j] : 1.0);
}

// LayerNorm (NEXT-4): y_j = (h_j - mean) / sqrt(var + eps) * w_j + b_j with
// mean and var (biased) over the n values, in two passes; w or b null means
// 1 or 0.
void layernorm(const double* h, int64_t n, const double* w, const double* b, double eps, double* y) {
  double sum = 0.0;
  for (int64_t j = 0; j < n; ++j) sum += h[j];
  const double mean = sum / (double)n;
  double ss = 0.0;
  for (int64_t j = 0; j < n; ++j) ss += (h[j] - mean) * (h[j] - mean);
  const double rstd = 1.0 / std::sqrt(ss / (double)n + eps);
  for (int64_t j = 0; j < n; ++j) y[j] = (h[j] - mean) * rstd * (w ? w[j] : 1.0) + (b ? b[j] : 0.0);
}

// Rotate-half RoPE ([FR] §2.2, second bullet): for j < n/2 the pair
// (v_j, v_{j+n/2}) is rotated by the angle whose cosine and sine are c_j, s_j.
void rope_rotate_half(double* v, int n, const float* c, const float* s) {
  const int half = n / 2;
  for (int j = 0; j < half; ++j) {
    const double a = v[j], b = v[j + half];
    const double cj = (double)c[j], sj = (double)s[j];
    v[j] = a * cj - b * sj;
    v[j + half] = b * cj + a * sj;
  }
}

// Gated activations ([FR] §二 steps 8-10: GELU(gate) * up; [FP] third
// technique: relu(gate)^2 * up; SiLU * up for the SwiGLU FFNs).
double act_fn(int act, double g) {
  switch (act) {
    case ACT_GELU_TANH: {
      const double k = std::sqrt(2.0 / M_PI);
      return 0.5 * g * (1.0 + std::tanh(k * (g + 0.044715 * g * g * g)));
    }
    case ACT_SILU:
      return g / (1.0 + std::exp(-g));
    case ACT_RELU2:
      return g > 0.0 ? g * g : 0.0;
    default:
      return NAN;
  }
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------- exports --
double oracle_f16_decode(uint16_t b) { return decode16(b, kF16); }
double oracle_bf16_decode(uint16_t b) { return decode16(b, kBF16); }
uint16_t oracle_f16_round(double hi, double lo) { return round16(hi, lo, kF16); }
uint16_t oracle_bf16_round(double hi, double lo) { return round16(hi, lo, kBF16); }
uint8_t oracle_e4m3_encode(double v) { return e4m3_encode(v); }
double oracle_e4m3_decode(uint8_t c) { return e4m3_decode(c); }
double oracle_act(int act, double g) { return act_fn(act, g); }

// 16-bit rounding of the exact sum of two 16-bit values (the residual add).
uint16_t oracle_add16(uint16_t x, uint16_t r, int dt) {
  const Fmt16 f = fmt_of(dt);
  double s, err;
  two_sum(decode16(x, f), decode16(r, f), &s, &err);
  return round16(s, err, f);
}

void oracle_quant_static(const double* y, int64_t n, double s, uint8_t* q) { quant_static(y, n, s, q); }
void oracle_quant_block128(const double* y, int64_t n, uint8_t* q, double* scales) {
  quant_block128(y, n, q, scales);
}
void oracle_rmsnorm(const double* h, int64_t n, const double* w, double eps, double* y) {
  rmsnorm(h, n, w, eps, y);
}
void oracle_rope_rotate_half(double* v, int n, const float* c, const float* s) { rope_rotate_half(v, n, c, s); }

// Op (a): residual add + RMSNorm + FP8 ([FR] §二 steps 1 and 7; §2.1 says
// the three element-wise steps share one read of the same input).
//   h = rn16(x + r) exactly rounded; residual_out = h; y = RMSNorm(h) in
//   fp64 (the norm reads the rounded h, as the unfused add -> norm pipeline
//   does); q = FP8(y) with the static scale or per-row block-128 scales.
//   residual_out may alias residual_in.  y_out (optional, [M, D]) receives
//   the fp64 y.  block_scales is [M, ceil(D/128)].  Returns 0, or -1 on a
//   bad argument.
int oracle_residual_rmsnorm_fp8(const uint16_t* x, const uint16_t* residual_in, uint16_t* residual_out,
                                const uint16_t* weight, uint8_t* out_fp8, double static_scale,
                                double* block_scales, double* y_out, int64_t M, int64_t D, double eps,
                                int dt, int qm) {
  if (M < 0 || D <= 0 || !x || !residual_in || !residual_out || !out_fp8) return -1;
  if (qm == Q_BLOCK128 && !block_scales) return -1;
  const Fmt16 f = fmt_of(dt);
  const int64_t nb = (D + 127) / 128;
  std::vector<double> h(D), w(D), y(D);
  if (weight)
    for (int64_t j = 0; j < D; ++j) w[j] = decode16(weight[j], f);
  for (int64_t i = 0; i < M; ++i) {
    for (int64_t j = 0; j < D; ++j) {
      double s, err;
      two_sum(decode16(x[i * D + j], f), decode16(residual_in[i * D + j], f), &s, &err);
      const uint16_t hb = round16(s, err, f);
      residual_out[i * D + j] = hb;
      h[j] = decode16(hb, f);
    }
    rmsnorm(h.data(), D, weight ? w.data() : nullptr, eps, y.data());
    if (y_out) std::memcpy(y_out + i * D, y.data(), sizeof(double) * D);
    if (qm == Q_STATIC)
      quant_static(y.data(), D, static_scale, out_fp8 + i * D);
    else
      quant_block128(y.data(), D, out_fp8 + i * D, block_scales + i * nb);
  }
  return 0;
}

// Op (b): packed QKV split + per-head q/k RMSNorm + rotate-half RoPE + Q
// staging write + KV-cache write ([FR] §2.2 first bullet: q_norm -> RoPE ->
// Q staging, k_norm -> RoPE -> KV cache; V passes through; [FR] §二 step 3).
//   qkv row i = [Q heads (Hq*hd) | K heads (Hkv*hd) | V heads (Hkv*hd)].
//   q_norm_w / k_norm_w ([hd], 16-bit) may each be null (no norm on that side).
//   cos/sin tables are [max_pos, hd/2] fp32; position p = positions[i].
//   q_out  [M, Hq, hd] receives the unrounded fp64 result.
//   k_cache [capacity, Hkv, hd] fp64, v_cache [capacity, Hkv, hd] 16-bit bits.
//   slots (optional, test convenience) stores row i at slots[i] instead of
//   at positions[i]; the rotation always uses positions[i].
//   A row whose position is outside [0, max_pos) or whose slot is outside
//   [0, capacity) is skipped and bit 0 of *status is set.
int oracle_qkv_norm_rope_kvcache(const uint16_t* qkv, const uint16_t* q_norm_w, const uint16_t* k_norm_w,
                                 const float* cos_tab, const float* sin_tab, const int32_t* positions,
                                 const int64_t* slots, double* q_out, double* k_cache, uint16_t* v_cache,
                                 int32_t* status, int64_t M, int64_t Hq, int64_t Hkv, int64_t hd,
                                 int64_t max_pos, int64_t capacity, double eps, int dt) {
  if (M < 0 || Hq <= 0 || Hkv <= 0 || hd <= 0 || hd % 2 != 0) return -1;
  if (!qkv || !cos_tab || !sin_tab || !positions || !q_out || !k_cache || !v_cache) return -1;
  const Fmt16 f = fmt_of(dt);
  const int64_t width = (Hq + 2 * Hkv) * hd;
  const int64_t half = hd / 2;
  std::vector<double> v(hd), wq(hd), wk(hd), y(hd);
  for (int64_t j = 0; j < hd; ++j) {
    if (q_norm_w) wq[j] = decode16(q_norm_w[j], f);
    if (k_norm_w) wk[j] = decode16(k_norm_w[j], f);
  }
  for (int64_t i = 0; i < M; ++i) {
    const int64_t p = positions[i];
    const int64_t slot = slots ? slots[i] : p;
    if (p < 0 || p >= max_pos || slot < 0 || slot >= capacity) {
      if (status) *status |= 1;
      continue;
    }
    const float* c = cos_tab + p * half;
    const float* s = sin_tab + p * half;
    const uint16_t* row = qkv + i * width;
    for (int64_t h = 0; h < Hq + Hkv; ++h) {
      const bool is_q = h < Hq;
      for (int64_t j = 0; j < hd; ++j) v[j] = decode16(row[h * hd + j], f);
      const uint16_t* nw = is_q ? q_norm_w : k_norm_w;
      if (nw) {
        rmsnorm(v.data(), hd, is_q ? wq.data() : wk.data(), eps, y.data());
        v = y;
      }
      rope_rotate_half(v.data(), (int)hd, c, s);
      double* dst = is_q ? q_out + (i * Hq + h) * hd : k_cache + (slot * Hkv + (h - Hq)) * hd;
      std::memcpy(dst, v.data(), sizeof(double) * hd);
    }
    for (int64_t g = 0; g < Hkv; ++g)
      std::memcpy(v_cache + (slot * Hkv + g) * hd, row + (Hq + Hkv + g) * hd, sizeof(uint16_t) * hd);
  }
  return 0;
}

// Op (c): gated activation on the interleaved gate/up buffer + FP8
// ([FP] third technique: adjacent (gate, up) pairs, even index = gate;
// [FR] §二 steps 8-10 GELU*up + quant; [FR4] Phase 2 block-128 FP8).
//   a_j = act(g_j) * u_j with g_j = gate_up[i, 2j], u_j = gate_up[i, 2j+1].
//   relu^2 takes g as given (sqrt(2) is already in the gate weights).
//   a_out (optional, [M, I]) receives the fp64 a.  block_scales is
//   [M, ceil(I/128)].
int oracle_gate_act_fp8(const uint16_t* gate_up, uint8_t* out_fp8, double static_scale, double* block_scales,
                        double* a_out, int64_t M, int64_t I, int act, int dt, int qm) {
  if (M < 0 || I <= 0 || !gate_up || !out_fp8) return -1;
  if (act < ACT_GELU_TANH || act > ACT_RELU2) return -1;
  if (qm == Q_BLOCK128 && !block_scales) return -1;
  const Fmt16 f = fmt_of(dt);
  const int64_t nb = (I + 127) / 128;
  std::vector<double> a(I);
  for (int64_t i = 0; i < M; ++i) {
    const uint16_t* row = gate_up + i * 2 * I;
    for (int64_t j = 0; j < I; ++j) {
      const double g = decode16(row[2 * j], f);
      const double u = decode16(row[2 * j + 1], f);
      a[j] = act_fn(act, g) * u;
    }
    if (a_out) std::memcpy(a_out + i * I, a.data(), sizeof(double) * I);
    if (qm == Q_STATIC)
      quant_static(a.data(), I, static_scale, out_fp8 + i * I);
    else
      quant_block128(a.data(), I, out_fp8 + i * I, block_scales + i * nb);
  }
  return 0;
}

// NEXT-1: gated residual + AdaRMSNorm modulation + FP8 ([FR] §三: the Pi0.5
// decoder's cross-layer kernel fuses gate multiply, residual add, AdaRMSNorm
// modulation, FP8 quantisation and descale, 6 ops -> 1, run 180 times per
// decode).  Reading (the pages give no formula; the adaptive RMSNorm of
// diffusion/flow-matching transformers):
//   c        = row / rows_per_cond (one condition per group of rows)
//   h        = rn16(r + g_c * x), the exact value rounded once
//   y        = h * rstd * (1 + scale_c) + shift_c, rstd = 1/sqrt(mean(h^2)+eps)
//   out_fp8  = FP8(y) as in op (a) (static or block-128)
// gate / scale / shift are [ceil(M / rows_per_cond), D] 16-bit; NULL gate
// means 1, NULL scale or shift means 0.  residual_out may alias residual_in.
int oracle_gate_residual_adarms_fp8(const uint16_t* x, const uint16_t* gate, const uint16_t* residual_in,
                                    uint16_t* residual_out, const uint16_t* scale, const uint16_t* shift,
                                    uint8_t* out_fp8, double static_scale, double* block_scales, double* y_out,
                                    int64_t M, int64_t D, int64_t rows_per_cond, double eps, int dt, int qm) {
  if (M < 0 || D <= 0 || rows_per_cond <= 0 || !x || !residual_in || !residual_out || !out_fp8) return -1;
  if (qm == Q_BLOCK128 && !block_scales) return -1;
  const Fmt16 f = fmt_of(dt);
  const int64_t nb = (D + 127) / 128;
  std::vector<double> h(D), y(D);
  for (int64_t i = 0; i < M; ++i) {
    const int64_t c = i / rows_per_cond;
    for (int64_t j = 0; j < D; ++j) {
      const double g = gate ? decode16(gate[c * D + j], f) : 1.0;
      const double gx = g * decode16(x[i * D + j], f);  // exact: two 16-bit significands
      double s, err;
      two_sum(decode16(residual_in[i * D + j], f), gx, &s, &err);
      const uint16_t hb = round16(s, err, f);
      residual_out[i * D + j] = hb;
      h[j] = decode16(hb, f);
    }
    rmsnorm(h.data(), D, nullptr, eps, y.data());
    for (int64_t j = 0; j < D; ++j) {
      const double sc = scale ? decode16(scale[c * D + j], f) : 0.0;
      const double sh = shift ? decode16(shift[c * D + j], f) : 0.0;
      y[j] = y[j] * (1.0 + sc) + sh;
    }
    if (y_out) std::memcpy(y_out + i * D, y.data(), sizeof(double) * D);
    if (qm == Q_STATIC)
      quant_static(y.data(), D, static_scale, out_fp8 + i * D);
    else
      quant_block128(y.data(), D, out_fp8 + i * D, block_scales + i * nb);
  }
  return 0;
}

// NEXT-2: op (b) with the attention's Q preparation folded in and an
// optional FP8 KV cache ([FR] §2.2 first bullet for op (b); the "sm89 / 5060
// Ti" port's step 10, FA2 prepare_q fused into RoPE).  Reading (the pages
// name the fusion only): prepare_q multiplies Q by the attention's softmax
// scale q_scale and may lay Q out head-major for the attention kernel; the
// FP8 cache holds e4m3 codes with one static dequantisation scale per tensor.
//   q        = rope(norm(q_head)) * q_scale (fp64, unrounded), stored at
//              q_out[i, h, :] (q_head_major == 0) or q_out[h, i, :] (== 1);
//   kv_fp8 == 0: k_cache (fp64) and v_cache (16-bit) exactly as op (b);
//   kv_fp8 == 1: k_cache8[slot, g, :] = e4m3(fp32(k) / fp32(k_scale)),
//                v_cache8[slot, g, :] = e4m3(fp32(v) / fp32(v_scale)), the
//                FP8 decision taken in fp32 as for the other FP8 outputs.
// Positions outside [0, max_pos) or slots outside [0, capacity) skip the row
// and set status bit 0, as op (b).
int oracle_qkv_norm_rope_prepq_kvcache(const uint16_t* qkv, const uint16_t* q_norm_w, const uint16_t* k_norm_w,
                                       const float* cos_tab, const float* sin_tab, const int32_t* positions,
                                       const int64_t* slots, double* q_out, double* k_cache, uint16_t* v_cache, uint8_t* k_cache8,
                                       uint8_t* v_cache8, int32_t* status, int64_t M, int64_t Hq, int64_t Hkv,
                                       int64_t hd, int64_t max_pos, int64_t capacity, double eps, int dt,
                                       double q_scale, int q_head_major, int kv_fp8, double k_scale,
                                       double v_scale) {
  if (M < 0 || Hq <= 0 || Hkv <= 0 || hd <= 0 || hd % 2 != 0) return -1;
  if (!qkv || !cos_tab || !sin_tab || !positions || !q_out) return -1;
  if (kv_fp8 ? (!k_cache8 || !v_cache8) : (!k_cache || !v_cache)) return -1;
  const Fmt16 f = fmt_of(dt);
  const int64_t width = (Hq + 2 * Hkv) * hd;
  const int64_t half = hd / 2;
  const float ks32 = (float)k_scale, vs32 = (float)v_scale;
  std::vector<double> v(hd), wq(hd), wk(hd), y(hd);
  for (int64_t j = 0; j < hd; ++j) {
    if (q_norm_w) wq[j] = decode16(q_norm_w[j], f);
    if (k_norm_w) wk[j] = decode16(k_norm_w[j], f);
  }
  for (int64_t i = 0; i < M; ++i) {
    const int64_t p = positions[i];
    // slots (test use only) stores row i's cache rows at slots[i] instead of
    // at p, so a sample of a large batch can use a compact cache.
    const int64_t slot = slots ? slots[i] : p;
    if (p < 0 || p >= max_pos || slot < 0 || slot >= capacity) {
      if (status) *status |= 1;
      continue;
    }
    const float* c = cos_tab + p * half;
    const float* s = sin_tab + p * half;
    const uint16_t* row = qkv + i * width;
    for (int64_t h = 0; h < Hq + Hkv; ++h) {
      const bool is_q = h < Hq;
      for (int64_t j = 0; j < hd; ++j) v[j] = decode16(row[h * hd + j], f);
      const uint16_t* nw = is_q ? q_norm_w : k_norm_w;
      if (nw) {
        rmsnorm(v.data(), hd, is_q ? wq.data() : wk.data(), eps, y.data());
        v = y;
      }
      rope_rotate_half(v.data(), (int)hd, c, s);
      if (is_q) {
        double* dst = q_head_major ? q_out + (h * M + i) * hd : q_out + (i * Hq + h) * hd;
        for (int64_t j = 0; j < hd; ++j) dst[j] = v[j] * q_scale;
      } else if (kv_fp8) {
        uint8_t* dst = k_cache8 + (slot * Hkv + (h - Hq)) * hd;
        for (int64_t j = 0; j < hd; ++j) dst[j] = quant_fp32(v[j], ks32);
      } else {
        std::memcpy(k_cache + (slot * Hkv + (h - Hq)) * hd, v.data(), sizeof(double) * hd);
      }
    }
    for (int64_t g = 0; g < Hkv; ++g) {
      const uint16_t* src = row + (Hq + Hkv + g) * hd;
      if (kv_fp8) {
        uint8_t* dst = v_cache8 + (slot * Hkv + g) * hd;
        for (int64_t j = 0; j < hd; ++j) dst[j] = quant_fp32(decode16(src[j], f), vs32);
      } else {
        std::memcpy(v_cache + (slot * Hkv + g) * hd, src, sizeof(uint16_t) * hd);
      }
    }
  }
  return 0;
}

// ------------------------------------------------------------- NEXT-3 --
uint8_t oracle_e2m1_encode(double v) { return e2m1_encode(v); }
double oracle_e2m1_decode(uint8_t c) { return e2m1_decode(c); }
int64_t oracle_sf_swizzle_offset(int64_t r, int64_t c, int64_t n_cols) { return sf_swizzle_offset(r, c, n_cols); }
void oracle_quant_nvfp4_row(const double* y, int64_t n, float gs, uint8_t* packed, uint8_t* sf) {
  quant_nvfp4_row(y, n, gs, packed, sf);
}

// Op (a) with an NVFP4 output ("residual_add_rms_norm_to_nvfp4"): h and y as
// op (a); out_fp4 [M, D/2] packed e2m1, sf [M, D/16] row-major e4m3.
int oracle_residual_rmsnorm_nvfp4(const uint16_t* x, const uint16_t* residual_in, uint16_t* residual_out,
                                  const uint16_t* weight, uint8_t* out_fp4, uint8_t* sf, double global_scale,
                                  double* y_out, int64_t M, int64_t D, double eps, int dt) {
  if (M < 0 || D <= 0 || D % 16 != 0 || !x || !residual_in || !residual_out || !out_fp4 || !sf) return -1;
  const Fmt16 f = fmt_of(dt);
  std::vector<double> h(D), w(D), y(D);
  if (weight)
    for (int64_t j = 0; j < D; ++j) w[j] = decode16(weight[j], f);
  for (int64_t i = 0; i < M; ++i) {
    for (int64_t j = 0; j < D; ++j) {
      double s, err;
      two_sum(decode16(x[i * D + j], f), decode16(residual_in[i * D + j], f), &s, &err);
      const uint16_t hb = round16(s, err, f);
      residual_out[i * D + j] = hb;
      h[j] = decode16(hb, f);
    }
    rmsnorm(h.data(), D, weight ? w.data() : nullptr, eps, y.data());
    if (y_out) std::memcpy(y_out + i * D, y.data(), sizeof(double) * D);
    quant_nvfp4_row(y.data(), D, (float)global_scale, out_fp4 + i * D / 2, sf + i * D / 16);
  }
  return 0;
}

// Op (c) with an NVFP4 output ("silu_mul_merged_grouped32"): a as op (c);
// out_fp4 [M, I/2] packed e2m1, sf [M, I/16] row-major e4m3.
int oracle_gate_act_nvfp4(const uint16_t* gate_up, uint8_t* out_fp4, uint8_t* sf, double global_scale,
                          double* a_out, int64_t M, int64_t I, int act, int dt) {
  if (M < 0 || I <= 0 || I % 16 != 0 || !gate_up || !out_fp4 || !sf) return -1;
  if (act < ACT_GELU_TANH || act > ACT_RELU2) return -1;
  const Fmt16 f = fmt_of(dt);
  std::vector<double> a(I);
  for (int64_t i = 0; i < M; ++i) {
    const uint16_t* row = gate_up + i * 2 * I;
    for (int64_t j = 0; j < I; ++j) a[j] = act_fn(act, decode16(row[2 * j], f)) * decode16(row[2 * j + 1], f);
    if (a_out) std::memcpy(a_out + i * I, a.data(), sizeof(double) * I);
    quant_nvfp4_row(a.data(), I, (float)global_scale, out_fp4 + i * I / 2, sf + i * I / 16);
  }
  return 0;
}

// ------------------------------------------------------------- NEXT-4 --
void oracle_layernorm(const double* h, int64_t n, const double* w, const double* b, double eps, double* y) {
  layernorm(h, n, w, b, eps, y);
}

// Op (a) with LayerNorm (the ViT "add_layer_norm" producer): h as op (a);
// y = LayerNorm(h) with weight / bias ([D] 16-bit, each optional); output
// FP8 (qm 0 / 1 as op (a)) or NVFP4 (out_fp4 [M, D/2], sf [M, D/16], gs).
int oracle_residual_layernorm_quant(const uint16_t* x, const uint16_t* residual_in, uint16_t* residual_out,
                                    const uint16_t* weight, const uint16_t* bias, uint8_t* out_q, double static_scale,
                                    double* block_scales, uint8_t* sf, double global_scale, double* y_out, int64_t M,
                                    int64_t D, double eps, int dt, int mode) {
  // mode 0: FP8 static, 1: FP8 block-128, 2: NVFP4
  if (M < 0 || D <= 0 || !x || !residual_in || !residual_out || !out_q) return -1;
  if ((mode == 1 && !block_scales) || (mode == 2 && (!sf || D % 16 != 0))) return -1;
  const Fmt16 f = fmt_of(dt);
  const int64_t nb = (D + 127) / 128;
  std::vector<double> h(D), w(D), b(D), y(D);
  for (int64_t j = 0; j < D; ++j) {
    if (weight) w[j] = decode16(weight[j], f);
    if (bias) b[j] = decode16(bias[j], f);
  }
  for (int64_t i = 0; i < M; ++i) {
    for (int64_t j = 0; j < D; ++j) {
      double s, err;
      two_sum(decode16(x[i * D + j], f), decode16(residual_in[i * D + j], f), &s, &err);
      const uint16_t hb = round16(s, err, f);
      residual_out[i * D + j] = hb;
      h[j] = decode16(hb, f);
    }
    layernorm(h.data(), D, weight ? w.data() : nullptr, bias ? b.data() : nullptr, eps, y.data());
    if (y_out) std::memcpy(y_out + i * D, y.data(), sizeof(double) * D);
    if (mode == 0)
      quant_static(y.data(), D, static_scale, out_q + i * D);
    else if (mode == 1)
      quant_block128(y.data(), D, out_q + i * D, block_scales + i * nb);
    else
      quant_nvfp4_row(y.data(), D, (float)global_scale, out_q + i * D / 2, sf + i * D / 16);
  }
  return 0;
}

// Op (b) with per-head LayerNorm on Q and K (the Chameleon prefill kernel:
// LayerNorm(Q) + LayerNorm(K) + rotate-half RoPE, [FR] §2.2 second bullet).
// q_w / q_b are [Hq, hd], k_w / k_b [Hkv, hd] (per-head affine), each
// optional; everything else as op (b).
int oracle_qkv_layernorm_rope_kvcache(const uint16_t* qkv, const uint16_t* q_w, const uint16_t* q_b,
                                      const uint16_t* k_w, const uint16_t* k_b, const float* cos_tab,
                                      const float* sin_tab, const int32_t* positions, const int64_t* slots,
                                      double* q_out, double* k_cache, uint16_t* v_cache, int32_t* status, int64_t M,
                                      int64_t Hq, int64_t Hkv, int64_t hd, int64_t max_pos, int64_t capacity,
                                      double eps, int dt) {
  if (M < 0 || Hq <= 0 || Hkv <= 0 || hd <= 0 || hd % 2 != 0) return -1;
  if (!qkv || !cos_tab || !sin_tab || !positions || !q_out || !k_cache || !v_cache) return -1;
  const Fmt16 f = fmt_of(dt);
  const int64_t width = (Hq + 2 * Hkv) * hd;
  const int64_t half = hd / 2;
  std::vector<double> v(hd), w(hd), b(hd), y(hd);
  for (int64_t i = 0; i < M; ++i) {
    const int64_t p = positions[i];
    const int64_t slot = slots ? slots[i] : p;
    if (p < 0 || p >= max_pos || slot < 0 || slot >= capacity) {
      if (status) *status |= 1;
      continue;
    }
    const float* c = cos_tab + p * half;
    const float* s = sin_tab + p * half;
    const uint16_t* row = qkv + i * width;
    for (int64_t h = 0; h < Hq + Hkv; ++h) {
      const bool is_q = h < Hq;
      const int64_t hh = is_q ? h : h - Hq;
      const uint16_t* pw = is_q ? q_w : k_w;
      const uint16_t* pb = is_q ? q_b : k_b;
      for (int64_t j = 0; j < hd; ++j) {
        v[j] = decode16(row[h * hd + j], f);
        if (pw) w[j] = decode16(pw[hh * hd + j], f);
        if (pb) b[j] = decode16(pb[hh * hd + j], f);
      }
      layernorm(v.data(), hd, pw ? w.data() : nullptr, pb ? b.data() : nullptr, eps, y.data());
      rope_rotate_half(y.data(), (int)hd, c, s);
      double* dst = is_q ? q_out + (i * Hq + h) * hd : k_cache + (slot * Hkv + hh) * hd;
      std::memcpy(dst, y.data(), sizeof(double) * hd);
    }
    for (int64_t g = 0; g < Hkv; ++g)
      std::memcpy(v_cache + (slot * Hkv + g) * hd, row + (Hq + Hkv + g) * hd, sizeof(uint16_t) * hd);
  }
  return 0;
}

}  // extern "C"
