// Offline weight preparation on the host (not on the forward path).
//
// PRQuant (Permutation Residual Quantization), §4 Method:
//   "Offline scaling and channel reordering" -- the k input channels of W with the largest
//   MXFP4 quantization error move to a contiguous tail (the AWQ scaling is the identity here);
//   "Offline residual augmentation" -- R_W = W~_tail - Q(W~_tail), and the GEMM weight is
//   Q([W~, R_W]) with reduction width C + k.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <string>
#include <vector>

#include "qlinear.h"

namespace {

float bf16_to_f32(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint32_t f32_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

// E2M1 code of an exactly-scaled value: nearest of {0,.5,1,1.5,2,3,4,6}, ties to the even code,
// saturating; sign bit from the input.
uint8_t e2m1_code(float v) {
  static const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
  const float a = std::min(std::fabs(v), 6.0f);
  int best = 0;
  for (int c = 1; c < 8; ++c) {
    const float dc = std::fabs(a - mag[c]), db = std::fabs(a - mag[best]);
    if (dc < db || (dc == db && (c & 1) == 0)) best = c;
  }
  return static_cast<uint8_t>(best | (std::signbit(v) ? 8 : 0));
}

float e2m1_value(uint8_t c) {
  static const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
  const float m = mag[c & 7];
  return (c & 8) ? -m : m;
}

// MXFP4 quantization of one row of fp32 values (each exactly representable), blocks of 32.
void quant_row_mx(const float* x, int64_t K, uint8_t* codes, uint8_t* sbytes) {
  for (int64_t b = 0; b < K / 32; ++b) {
    float amax = 0.f;
    for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(x[b * 32 + i]));
    const int E = static_cast<int>((f32_bits(amax) >> 23) & 0xFF);
    const int e = (E == 0) ? -127 : std::max(E - 129, -127);
    sbytes[b] = static_cast<uint8_t>(e + 127);
    const float inv = std::ldexp(1.0f, -e);
    for (int i = 0; i < 32; ++i) codes[b * 32 + i] = e2m1_code(x[b * 32 + i] * inv);
  }
}

// MXFP4 quantization of one row with the E8M0-W local block-scale search (PRQuant §5.3): per
// 32-block the OCP exponent e0 and its neighbours e0 + 1, e0 - 1 (clamped to [-127, 127]) are
// tried in that order with the same element rule; the block keeps the first with the smallest
// sum of squared errors (double, summed in element order; a later one only if strictly better).
void quant_row_mx_search(const float* x, int64_t K, uint8_t* codes, uint8_t* sbytes) {
  for (int64_t b = 0; b < K / 32; ++b) {
    float amax = 0.f;
    for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(x[b * 32 + i]));
    const int E = static_cast<int>((f32_bits(amax) >> 23) & 0xFF);
    const int e0 = (E == 0) ? -127 : std::max(E - 129, -127);
    int best_e = e0;
    double best_err = 0;
    uint8_t best[32], cand[32];
    for (int t = 0; t < 3; ++t) {
      const int e = std::min(127, std::max(-127, e0 + (t == 0 ? 0 : t == 1 ? 1 : -1)));
      double err = 0;
      for (int i = 0; i < 32; ++i) {
        const double v = static_cast<double>(x[b * 32 + i]);
        cand[i] = e2m1_code(static_cast<float>(std::ldexp(v, -e)));
        const double d = v - static_cast<double>(e2m1_value(cand[i])) * std::ldexp(1.0, e);
        err += d * d;
      }
      if (t == 0 || err < best_err) {
        best_err = err;
        best_e = e;
        std::memcpy(best, cand, 32);
      }
    }
    sbytes[b] = static_cast<uint8_t>(best_e + 127);
    std::memcpy(codes + b * 32, best, 32);
  }
}

}  // namespace

extern "C" ql_status qlinear_prepare_prquant_ex(const uint16_t* w_bf16, int64_t N, int64_t C,
                                                int32_t k, int32_t scale_search, int32_t* perm_out,
                                                uint8_t* codes_out, uint8_t* scales_out);

extern "C" ql_status qlinear_prepare_prquant(const uint16_t* w_bf16, int64_t N, int64_t C,
                                             int32_t k, int32_t* perm_out, uint8_t* codes_out,
                                             uint8_t* scales_out) {
  return qlinear_prepare_prquant_ex(w_bf16, N, C, k, 0, perm_out, codes_out, scales_out);
}

extern "C" ql_status qlinear_prepare_prquant_ex(const uint16_t* w_bf16, int64_t N, int64_t C,
                                                int32_t k, int32_t scale_search, int32_t* perm_out,
                                                uint8_t* codes_out, uint8_t* scales_out) {
  auto quant_row = scale_search ? quant_row_mx_search : quant_row_mx;
  if (w_bf16 == nullptr || perm_out == nullptr || codes_out == nullptr || scales_out == nullptr)
    return QL_ERR_INVALID_ARG;
  if (N <= 0 || C <= 0 || k <= 0 || k > C) return QL_ERR_INVALID_ARG;
  if (C % 128 != 0 || k % 128 != 0) return QL_ERR_UNSUPPORTED;
  const int64_t Kp = C + k;
  // 1. per-column squared MXFP4 error of W, summed over rows in row order
  std::vector<double> err(C, 0.0);
  {
    std::vector<float> row(C);
    std::vector<uint8_t> codes(C), sb(C / 32);
    for (int64_t n = 0; n < N; ++n) {
      for (int64_t c = 0; c < C; ++c) row[c] = bf16_to_f32(w_bf16[n * C + c]);
      quant_row(row.data(), C, codes.data(), sb.data());
      for (int64_t c = 0; c < C; ++c) {
        const double d = static_cast<double>(row[c]) -
                         static_cast<double>(e2m1_value(codes[c])) * std::ldexp(1.0, sb[c / 32] - 127);
        err[c] += d * d;
      }
    }
  }
  // 2. top-k channels (ties to the lower index), then the permutation
  std::vector<int32_t> order(C);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int32_t a, int32_t b) { return err[a] > err[b]; });
  std::vector<char> is_tail(C, 0);
  for (int32_t i = 0; i < k; ++i) is_tail[order[i]] = 1;
  int32_t pos = 0;
  for (int32_t c = 0; c < C; ++c)
    if (!is_tail[c]) perm_out[pos++] = c;
  for (int32_t c = 0; c < C; ++c)
    if (is_tail[c]) perm_out[pos++] = c;
  // 3. quantize the permuted weight and its tail residual
  std::vector<float> row(C), res(k);
  std::vector<uint8_t> codes(Kp), sb(Kp / 32);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < C; ++j) row[j] = bf16_to_f32(w_bf16[n * C + perm_out[j]]);
    quant_row(row.data(), C, codes.data(), sb.data());
    for (int32_t j = 0; j < k; ++j) {
      const int64_t c = C - k + j;
      res[j] = row[c] - e2m1_value(codes[c]) * std::ldexp(1.0f, sb[c / 32] - 127);  // exact
    }
    quant_row(res.data(), k, codes.data() + C, sb.data() + C / 32);
    for (int64_t j = 0; j < Kp / 2; ++j)
      codes_out[n * (Kp / 2) + j] =
          static_cast<uint8_t>((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
    std::memcpy(scales_out + n * (Kp / 32), sb.data(), Kp / 32);
  }
  return QL_OK;
}

// MXCode PreScale VQ (MXCode abstract; Table 1 row E4M3-B16-FP4): the E4M3 block scales and the
// FP32 tensor scale are taken from W first; each 4-vector of W / (block scale * tensor scale) is
// then replaced by the index of the nearest entry of its QBlock's E2M1 codebook.
namespace {

// Finite non-negative E4M3 values, codes 0x00..0x7E, ascending.
struct E4m3Table {
  float v[127];
  E4m3Table() {
    for (int b = 0; b < 127; ++b) {
      const int e = b >> 3, m = b & 7;
      v[b] = e == 0 ? std::ldexp(static_cast<float>(m), -9)
                    : std::ldexp(static_cast<float>(8 + m), e - 10);
    }
  }
  // nearest, ties to the even code, saturating at 448
  uint8_t encode(float r) const {
    if (!(r > 0.f)) return 0;
    if (r >= v[126]) return 126;
    int lo = 0, hi = 126;
    while (hi - lo > 1) {
      const int mid = (lo + hi) / 2;
      if (v[mid] <= r) lo = mid; else hi = mid;
    }
    const float dlo = r - v[lo], dhi = v[hi] - r;
    if (dhi < dlo) return static_cast<uint8_t>(hi);
    if (dlo < dhi) return static_cast<uint8_t>(lo);
    return static_cast<uint8_t>((lo % 2 == 0) ? lo : hi);
  }
};

}  // namespace

extern "C" ql_status qlinear_prepare_vq_prescale(const uint16_t* w_bf16, int64_t N, int64_t K,
                                                 const uint8_t* codebooks, int32_t qn, int32_t qk,
                                                 float* ts_out, uint8_t* scales_out,
                                                 uint8_t* idx_out) {
  if (w_bf16 == nullptr || codebooks == nullptr || ts_out == nullptr || scales_out == nullptr ||
      idx_out == nullptr)
    return QL_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || qn != 64 || qk != 64 || N % qn != 0 || K % qk != 0)
    return QL_ERR_UNSUPPORTED;
  static const E4m3Table tab;
  float amax = 0.f;
  for (int64_t i = 0; i < N * K; ++i) amax = std::max(amax, std::fabs(bf16_to_f32(w_bf16[i])));
  const float ts = amax == 0.f ? 1.f : amax / 2688.0f;
  *ts_out = ts;
  const int64_t QC = K / qk;
  // E2M1 values of every codebook entry: [QR][QC][256][4]
  static const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < N; ++n) {
    std::vector<float> v(K);
    for (int64_t b = 0; b < K / 16; ++b) {
      float am = 0.f;
      for (int i = 0; i < 16; ++i) am = std::max(am, std::fabs(bf16_to_f32(w_bf16[n * K + b * 16 + i])));
      const float t = am / 6.0f;
      const float r = t / ts;
      const uint8_t s = tab.encode(r);
      scales_out[n * (K / 16) + b] = s;
      const float S = tab.v[s] * ts;
      for (int i = 0; i < 16; ++i)
        v[b * 16 + i] = S == 0.f ? 0.f : bf16_to_f32(w_bf16[n * K + b * 16 + i]) / S;
    }
    const int64_t qr = n / qn;
    for (int64_t j = 0; j < K / 4; ++j) {
      const uint8_t* cb = codebooks + ((qr * QC + (j * 4) / qk) * 256) * 2;
      int best = 0;
      double bestd = 0;
      for (int e = 0; e < 256; ++e) {
        double d = 0;
        for (int i = 0; i < 4; ++i) {
          const uint8_t c = (cb[e * 2 + i / 2] >> (4 * (i & 1))) & 0xF;
          const double cv = (c & 8) ? -mag[c & 7] : mag[c & 7];
          const double diff = static_cast<double>(v[j * 4 + i]) - cv;
          d += diff * diff;
        }
        if (e == 0 || d < bestd) { bestd = d; best = e; }
      }
      idx_out[n * (K / 4) + j] = static_cast<uint8_t>(best);
    }
  }
  return QL_OK;
}

// MosaicQuant-style INT4 dense base + block-sparse INT4 residual ("Dense Base and Sparse
// Residuals", "Activation-aware Delta-Hessian Block Selection").  Per (row, 128-group) the base
// scale is fp16(amax/7) and codes clamp(rint(w/s), -7, 7); dW = W - base; the score of a 16 x 128
// block is the sum over its rows, then columns, of abar_k |dW| with abar_k = mean_t |x_t,k| over
// the calibration rows; the round(density * blocks) best blocks (ties to the lower id) keep a
// residual quantized like the base on fp32(dW).
namespace {

uint16_t f32_to_f16_rne(float f) {
  const uint32_t x = f32_bits(f);
  const uint32_t sign = (x >> 16) & 0x8000u;
  if ((x & 0x7FFFFFFFu) == 0) return static_cast<uint16_t>(sign);
  const int exp = static_cast<int>((x >> 23) & 0xFF) - 127 + 15;
  uint32_t mant = x & 0x7FFFFFu;
  if (exp >= 31) return static_cast<uint16_t>(sign | 0x7C00u);           // overflow -> inf
  if (exp <= 0) {                                                          // fp16 subnormal
    if (exp < -10) return static_cast<uint16_t>(sign);
    mant |= 0x800000u;
    const int shift = 14 - exp;
    uint32_t h = mant >> shift;
    const uint32_t rem = mant & ((1u << shift) - 1u), half = 1u << (shift - 1);
    if (rem > half || (rem == half && (h & 1u))) ++h;
    return static_cast<uint16_t>(sign | h);
  }
  uint32_t h = sign | (static_cast<uint32_t>(exp) << 10) | (mant >> 13);
  const uint32_t rem = mant & 0x1FFFu;
  if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) ++h;
  return static_cast<uint16_t>(h);
}

float f16_to_f32(uint16_t h) {
  const uint32_t s = (h & 0x8000u) << 16, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  if (e == 0) {
    const float v = std::ldexp(static_cast<float>(m), -24);
    return s ? -v : v;
  }
  if (e == 31) {
    uint32_t u = s | 0x7F800000u | (m << 13);
    float f;
    std::memcpy(&f, &u, 4);
    return f;
  }
  uint32_t u = s | ((e + 112) << 23) | (m << 13);
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// INT4 codes of one 128-group with an fp16 scale; returns the scale bits.
uint16_t quant_group_int4(const float* w, int8_t* q) {
  float amax = 0.f;
  for (int i = 0; i < 128; ++i) amax = std::max(amax, std::fabs(w[i]));
  const uint16_t s16 = f32_to_f16_rne(amax / 7.0f);
  const float sf = f16_to_f32(s16);
  for (int i = 0; i < 128; ++i) {
    if (sf == 0.f) { q[i] = 0; continue; }
    const float r = std::nearbyint(w[i] / sf);
    q[i] = static_cast<int8_t>(std::min(7.f, std::max(-7.f, r)));
  }
  return s16;
}

}  // namespace

extern "C" ql_status qlinear_prepare_int4_bsr(const uint16_t* w_bf16, int64_t N, int64_t K,
                                              const uint16_t* x_calib_bf16, int64_t T,
                                              float density, uint8_t* codes_out,
                                              uint16_t* scales_out, int32_t* rowptr_out,
                                              int16_t* col_out, uint8_t* rcodes_out,
                                              uint16_t* rscales_out, int32_t capacity,
                                              int32_t* nnzb_out) {
  if (!w_bf16 || !x_calib_bf16 || !codes_out || !scales_out || !rowptr_out || !col_out ||
      !rcodes_out || !rscales_out || !nnzb_out)
    return QL_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || T <= 0 || N % 16 != 0 || K % 128 != 0 || !(density >= 0.f && density <= 1.f))
    return QL_ERR_INVALID_ARG;
  const int64_t G = K / 128, NB = N / 16;
  std::vector<double> dw(static_cast<size_t>(N) * K);
  std::vector<float> row(K);
  std::vector<int8_t> q(128);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) row[k] = bf16_to_f32(w_bf16[n * K + k]);
    for (int64_t g = 0; g < G; ++g) {
      const uint16_t s16 = quant_group_int4(&row[g * 128], q.data());
      scales_out[n * G + g] = s16;
      const double sf = f16_to_f32(s16);
      for (int i = 0; i < 128; ++i) {
        const int64_t k = g * 128 + i;
        dw[n * K + k] = static_cast<double>(row[k]) - static_cast<double>(q[i]) * sf;
        const uint8_t nib = static_cast<uint8_t>(q[i]) & 0xF;
        uint8_t& b = codes_out[n * (K / 2) + k / 2];
        b = (k & 1) ? static_cast<uint8_t>((b & 0x0F) | (nib << 4)) : nib;
      }
    }
  }
  std::vector<double> abar(K, 0.0);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t k = 0; k < K; ++k) abar[k] += std::fabs(static_cast<double>(bf16_to_f32(x_calib_bf16[t * K + k])));
  for (int64_t k = 0; k < K; ++k) abar[k] /= static_cast<double>(T);
  std::vector<double> score(static_cast<size_t>(NB) * G, 0.0);
  for (int64_t nb = 0; nb < NB; ++nb)
    for (int64_t g = 0; g < G; ++g) {
      double s = 0.0;
      for (int r = 0; r < 16; ++r)
        for (int i = 0; i < 128; ++i) {
          const int64_t k = g * 128 + i;
          s += std::fabs(dw[(nb * 16 + r) * K + k]) * abar[k];
        }
      score[nb * G + g] = s;
    }
  const int64_t keep = static_cast<int64_t>(std::llround(static_cast<double>(density) * NB * G));
  if (keep > capacity) return QL_ERR_INVALID_ARG;
  std::vector<int64_t> order(NB * G);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int64_t a, int64_t b) { return score[a] > score[b]; });
  std::vector<int64_t> sel(order.begin(), order.begin() + keep);
  std::sort(sel.begin(), sel.end());
  std::fill(rowptr_out, rowptr_out + NB + 1, 0);
  std::vector<float> seg(128);
  for (int64_t i = 0; i < keep; ++i) {
    const int64_t nb = sel[i] / G, g = sel[i] % G;
    rowptr_out[nb + 1] += 1;
    col_out[i] = static_cast<int16_t>(g);
    for (int r = 0; r < 16; ++r) {
      for (int j = 0; j < 128; ++j) seg[j] = static_cast<float>(dw[(nb * 16 + r) * K + g * 128 + j]);
      rscales_out[i * 16 + r] = quant_group_int4(seg.data(), q.data());
      for (int j = 0; j < 64; ++j)
        rcodes_out[(i * 16 + r) * 64 + j] = static_cast<uint8_t>((static_cast<uint8_t>(q[2 * j]) & 0xF) |
                                                                 ((static_cast<uint8_t>(q[2 * j + 1]) & 0xF) << 4));
    }
  }
  for (int64_t nb = 0; nb < NB; ++nb) rowptr_out[nb + 1] += rowptr_out[nb];
  *nnzb_out = static_cast<int32_t>(keep);
  return QL_OK;
}

// MXCode PostScale (MXCode abstract: "quantizes learned codebooks to MXFP4"): each QBlock's
// learned codebook (256 x 4 values) is quantized to E2M1 with one E4M3 scale for the whole
// codebook, relative to an FP32 tensor scale over all codebooks, so that every 16-block of the
// decoded weight in the QBlock carries that scale (an MX-native operand; no per-weight scales).
// Each 4-vector of W takes the nearest decoded entry (exact values, squared distance in double,
// ties to the lowest index).
extern "C" ql_status qlinear_prepare_vq_postscale(const uint16_t* w_bf16, int64_t N, int64_t K,
                                                  const float* centroids, int32_t qn, int32_t qk,
                                                  float* ts_out, uint8_t* codebooks_out,
                                                  uint8_t* qscales_out, uint8_t* idx_out) {
  if (w_bf16 == nullptr || centroids == nullptr || ts_out == nullptr || codebooks_out == nullptr ||
      qscales_out == nullptr || idx_out == nullptr)
    return QL_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || qn != 64 || qk != 64 || N % qn != 0 || K % qk != 0)
    return QL_ERR_UNSUPPORTED;
  static const E4m3Table tab;
  const int64_t QR = N / qn, QC = K / qk, nq = QR * QC;
  float amax_t = 0.f;
  for (int64_t i = 0; i < nq * 1024; ++i) amax_t = std::max(amax_t, std::fabs(centroids[i]));
  const float ts = amax_t == 0.f ? 1.f : amax_t / 2688.0f;
  *ts_out = ts;
  std::vector<double> vals(static_cast<size_t>(nq) * 1024);   // decoded entry values
  for (int64_t q = 0; q < nq; ++q) {
    const float* c = centroids + q * 1024;
    float am = 0.f;
    for (int i = 0; i < 1024; ++i) am = std::max(am, std::fabs(c[i]));
    const float t = am / 6.0f;
    const float r = t / ts;
    const uint8_t s = tab.encode(r);
    qscales_out[q] = s;
    const float S = tab.v[s] * ts;
    const double scale = static_cast<double>(tab.v[s]) * static_cast<double>(ts);
    uint8_t* cb = codebooks_out + q * 512;
    for (int e = 0; e < 256; ++e) {
      uint8_t code[4];
      for (int i = 0; i < 4; ++i) {
        const float x = c[e * 4 + i];
        code[i] = S == 0.f ? static_cast<uint8_t>(std::signbit(x) ? 8 : 0) : e2m1_code(x / S);
        vals[q * 1024 + e * 4 + i] = static_cast<double>(e2m1_value(code[i])) * scale;
      }
      cb[e * 2] = static_cast<uint8_t>((code[0] & 0xF) | (code[1] << 4));
      cb[e * 2 + 1] = static_cast<uint8_t>((code[2] & 0xF) | (code[3] << 4));
    }
  }
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < N; ++n) {
    const int64_t qr = n / qn;
    for (int64_t j = 0; j < K / 4; ++j) {
      const double* v = vals.data() + (qr * QC + (j * 4) / qk) * 1024;
      int best = 0;
      double bestd = 0;
      for (int e = 0; e < 256; ++e) {
        double d = 0;
        for (int i = 0; i < 4; ++i) {
          const double diff = static_cast<double>(bf16_to_f32(w_bf16[n * K + j * 4 + i])) - v[e * 4 + i];
          d += diff * diff;
        }
        if (e == 0 || d < bestd) { bestd = d; best = e; }
      }
      idx_out[n * (K / 4) + j] = static_cast<uint8_t>(best);
    }
  }
  return QL_OK;
}

// MXCode PreScale+ (MXCode abstract: PreScale's scales "further compressed using VQ"; appendix
// Table 4 caption: Ks = 256, ds = 8): the E4M3 block scales of PreScale, 8 consecutive along K,
// are replaced by the nearest of 256 scale vectors of a per-tensor scale codebook (squared
// distance of decoded scale values in double, ties to the lowest index); W is then normalised by
// the compressed scales and assigned as in PreScale.  Outputs: ts, the compressed scale bytes
// [N, K/16], the scale indices [N, K/128] and the weight indices [N, K/4].
extern "C" ql_status qlinear_prepare_vq_prescale_plus(const uint16_t* w_bf16, int64_t N, int64_t K,
                                                      const uint8_t* codebooks,
                                                      const uint8_t* scale_codebook, int32_t qn,
                                                      int32_t qk, float* ts_out,
                                                      uint8_t* scales_out, uint8_t* sidx_out,
                                                      uint8_t* idx_out) {
  if (w_bf16 == nullptr || codebooks == nullptr || scale_codebook == nullptr || ts_out == nullptr ||
      scales_out == nullptr || sidx_out == nullptr || idx_out == nullptr)
    return QL_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || qn != 64 || qk != 64 || N % qn != 0 || K % qk != 0 || K % 128 != 0)
    return QL_ERR_UNSUPPORTED;
  static const E4m3Table tab;
  float amax = 0.f;
  for (int64_t i = 0; i < N * K; ++i) amax = std::max(amax, std::fabs(bf16_to_f32(w_bf16[i])));
  const float ts = amax == 0.f ? 1.f : amax / 2688.0f;
  *ts_out = ts;
  const int64_t QC = K / qk, G16 = K / 16;
  static const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < N; ++n) {
    std::vector<uint8_t> s0(G16);
    for (int64_t b = 0; b < G16; ++b) {
      float am = 0.f;
      for (int i = 0; i < 16; ++i) am = std::max(am, std::fabs(bf16_to_f32(w_bf16[n * K + b * 16 + i])));
      const float t = am / 6.0f;
      s0[b] = tab.encode(t / ts);
    }
    for (int64_t g = 0; g < G16 / 8; ++g) {   // nearest scale vector
      int best = 0;
      double bestd = 0;
      for (int e = 0; e < 256; ++e) {
        double d = 0;
        for (int i = 0; i < 8; ++i) {
          const uint8_t cb = scale_codebook[e * 8 + i];
          const double diff = static_cast<double>(tab.v[s0[g * 8 + i] & 0x7F]) -
                              static_cast<double>(cb <= 126 ? tab.v[cb] : 0.f);
          d += diff * diff;
        }
        if (e == 0 || d < bestd) { bestd = d; best = e; }
      }
      sidx_out[n * (G16 / 8) + g] = static_cast<uint8_t>(best);
      for (int i = 0; i < 8; ++i) scales_out[n * G16 + g * 8 + i] = scale_codebook[best * 8 + i];
    }
    std::vector<float> v(K);
    for (int64_t b = 0; b < G16; ++b) {
      const uint8_t s = scales_out[n * G16 + b];
      const float S = (s <= 126 ? tab.v[s] : 0.f) * ts;
      for (int i = 0; i < 16; ++i)
        v[b * 16 + i] = S == 0.f ? 0.f : bf16_to_f32(w_bf16[n * K + b * 16 + i]) / S;
    }
    const int64_t qr = n / qn;
    for (int64_t j = 0; j < K / 4; ++j) {
      const uint8_t* cb = codebooks + ((qr * QC + (j * 4) / qk) * 256) * 2;
      int best = 0;
      double bestd = 0;
      for (int e = 0; e < 256; ++e) {
        double d = 0;
        for (int i = 0; i < 4; ++i) {
          const uint8_t c = (cb[e * 2 + i / 2] >> (4 * (i & 1))) & 0xF;
          const double cv = (c & 8) ? -mag[c & 7] : mag[c & 7];
          const double diff = static_cast<double>(v[j * 4 + i]) - cv;
          d += diff * diff;
        }
        if (e == 0 || d < bestd) { bestd = d; best = e; }
      }
      idx_out[n * (K / 4) + j] = static_cast<uint8_t>(best);
    }
  }
  return QL_OK;
}
