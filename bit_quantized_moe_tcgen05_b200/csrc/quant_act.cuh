// Online activation quantizers (HBM-bound, CUDA cores).
//
//  * quant_mx_e8m0_b32_kernel -- OCP-MX / MXFP4: per 32 elements along K a shared exponent
//    e = floor(log2 amax) - 2 (clamped to [-127,127], stored as the E8M0 byte e+127), elements
//    x * 2^-e rounded to nearest-even E2M1 and saturated at +-6.  PRQuant, §4 "Kernel design for
//    efficient inference" quantizes the reordered activation to MXFP4 once; the tail copy that
//    page appends is realised by the GEMM reading the same quantized tail twice.
//  * quant_e4m3_b16 kernels -- E4M3-B16-FP4 with an FP32 tensor scale (MXCode, Table 1).
//  * quant_int4_g128_kernel -- symmetric INT4 per (token, 128-group), fp32 scale amax/7
//    (MosaicQuant W4A4 INT4 path).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

namespace ql {

// Round an (exactly scaled) fp32 value to the nearest E2M1 code, ties to the even code,
// saturating at 6; the sign bit follows the input's sign bit.
__device__ __forceinline__ uint32_t e2m1_rne(float v) {
  const float a = fabsf(v);
  uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
               (a >= 3.5f) + (a > 5.0f);
  return c | ((__float_as_uint(v) >> 28) & 8u);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Offset of scale (row m, scale column j) in the tiled scale-factor layout used by the
// block-scaled MMA: 512-byte atoms of 128 rows x 4 scale columns, atoms ordered K-fastest;
// inside an atom, row m sits at (m%32)*16 + ((m/32)%4)*4 and column j at j%4.
__host__ __device__ __forceinline__ size_t sf_tiled_offset(int m, int j, int atoms_per_row) {
  const size_t atom = static_cast<size_t>(m >> 7) * atoms_per_row + (j >> 2);
  return atom * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (j & 3);
}

// One thread per 8 consecutive elements; four threads (one quad of lanes) share a 32-block.
// x: bf16 [M, K] with row stride ldx (elements).  codes: [M, K/2] bytes (row stride ldc),
// low nibble = even k.  Scales go to the plain [M, K/32] layout and/or the tiled layout.
// The first `nzero` ints of `zero_words` are cleared (split-K tile tickets of the GEMM that
// consumes this output).
__global__ void __launch_bounds__(256) quant_mx_e8m0_b32_kernel(
    const __nv_bfloat16* __restrict__ x, int M, int K, int ldx, uint8_t* __restrict__ codes,
    int ldc, uint8_t* __restrict__ scales_plain, int lds, uint8_t* __restrict__ scales_tiled,
    int sf_atoms_per_row, int* __restrict__ zero_words, int nzero) {
  const long gtid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (zero_words != nullptr && gtid < nzero) zero_words[gtid] = 0;
  const int groups = K >> 3;
  const long total = static_cast<long>(M) * groups;
  if (gtid >= total) return;  // total is a multiple of 4: quads stay whole
  const int m = static_cast<int>(gtid / groups);
  const int q = static_cast<int>(gtid - static_cast<long>(m) * groups);
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * ldx) + q);
  float f[8];
  bf16x8_to_f32(v, f);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
  const unsigned mask = __activemask();
  amax = fmaxf(amax, __shfl_xor_sync(mask, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(mask, amax, 2));
  // floor(log2 amax) from the fp32 exponent field; zero and fp32-subnormal amax give an
  // exponent at or below -127 and clamp to -127.  bf16 cannot exceed 2^128, so e <= 125.
  const int E = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF);
  const int e = (E == 0) ? -127 : max(E - 129, -127);
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, normal
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) packed |= e2m1_rne(f[i] * inv) << (4 * i);
  *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(m) * ldc + q * 4) = packed;
  if ((q & 3) == 0) {
    const uint8_t b = static_cast<uint8_t>(e + 127);
    const int j = q >> 2;
    if (scales_plain != nullptr) scales_plain[static_cast<size_t>(m) * lds + j] = b;
    if (scales_tiled != nullptr) scales_tiled[sf_tiled_offset(m, j, sf_atoms_per_row)] = b;
  }
}

}  // namespace ql
