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

}  // namespace

extern "C" ql_status qlinear_prepare_prquant(const uint16_t* w_bf16, int64_t N, int64_t C,
                                             int32_t k, int32_t* perm_out, uint8_t* codes_out,
                                             uint8_t* scales_out) {
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
      quant_row_mx(row.data(), C, codes.data(), sb.data());
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
    quant_row_mx(row.data(), C, codes.data(), sb.data());
    for (int32_t j = 0; j < k; ++j) {
      const int64_t c = C - k + j;
      res[j] = row[c] - e2m1_value(codes[c]) * std::ldexp(1.0f, sb[c / 32] - 127);  // exact
    }
    quant_row_mx(res.data(), k, codes.data() + C, sb.data() + C / 32);
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
