// Online activation quantizers (HBM-bound, CUDA cores).
//
//  * quant_mx_e8m0_b32_kernel -- OCP-MX / MXFP4: per 32 elements along K a shared exponent
//    e = floor(log2 amax) - 2 (clamped to [-127,127], stored as the E8M0 byte e+127), elements
//    x * 2^-e rounded to nearest-even E2M1 and saturated at +-6.  PRQuant, §4 "Kernel design for
//    efficient inference" quantizes the reordered activation to MXFP4 once and appends the
//    quantized tail: either the GEMM reads the same quantized tail twice (online), or this
//    kernel writes the tail blocks a second time behind the others (offline copy, "Activation
//    tail construction").
//  * quant_e4m3_b16 kernels -- E4M3-B16-FP4 with an FP32 tensor scale (MXCode, Table 1).
//  * quant_int4_g128_kernel -- symmetric INT4 per (token, 128-group), fp32 scale amax/7
//    (MosaicQuant W4A4 INT4 path).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "ptx.cuh"

namespace ql {

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
// Rows are grouped by the GEMM's token tiles of tile_rows rows (128, 160 or 256): tile t owns
// ceil(tile_rows / 128) consecutive 128-row atom groups, so that a tile's scales start on an atom
// boundary whatever its first row; with tile_rows = 128 or 256 this is plain 128-row grouping.
__host__ __device__ __forceinline__ size_t sf_tiled_offset(int m, int j, int atoms_per_row,
                                                           int tile_rows) {
  const int groups = (tile_rows + 127) >> 7;
  const int t = m / tile_rows, r = m - t * tile_rows;
  const size_t atom = static_cast<size_t>(t * groups + (r >> 7)) * atoms_per_row + (j >> 2);
  return atom * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (j & 3);
}

// Eight E2M1 codes from eight exactly-scaled fp32 values (RNE, satfinite) via the hardware
// conversion; element 2i lands in the low nibble.  The sign bits are or-ed in from the inputs so
// that negative values rounding to zero keep code 0x8 whatever the conversion does with zeros.
__device__ __forceinline__ uint32_t e2m1x8(const float (&f)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]), "f"(f[6]), "f"(f[7]));
  return out;
}

// Value of an E2M1 code (bit 3 = sign).
__device__ __forceinline__ float e2m1_code_value(uint32_t c) {
  const uint32_t m = c & 7u;
  const float mag = m < 2 ? 0.5f * static_cast<float>(m)
                          : __uint_as_float(((126u + (m >> 1)) << 23) | ((m & 1u) << 22));
  return (c & 8u) ? -mag : mag;
}

// Sign bits of eight bf16 values packed in four words (element 2i low half of word i) placed at
// bit 3 of each nibble of the matching code word.
__device__ __forceinline__ uint32_t bf16x8_sign_nibbles(const uint32_t (&w)[4]) {
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    s |= (((w[i] >> 12) & 0x8u) | ((w[i] >> 24) & 0x80u)) << (8 * i);
  return s;
}

// Online block Hadamard (CodeQuant's "had" variants: online Hadamard transforms during
// quantization; block 32, the MX block): the 32 values of one block, in fp32, through the
// Walsh-Hadamard butterfly in the order h = 1, 2, 4, 8, 16, each step (a, b) -> (a + b, a - b) a
// plain fp32 addition or subtraction, so the result is x . H_32 (Sylvester order, unnormalised;
// the weight carries H_32 / 32).
__device__ __forceinline__ void fwht32(float (&v)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1)
#pragma unroll
    for (int i = 0; i < 32; i += 2 * h)
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float a = v[j], b = v[j + h];
        v[j] = __fadd_rn(a, b);
        v[j + h] = __fsub_rn(a, b);
      }
}

// MX E8M0-B32 coding of 32 fp32 values (each exactly scalable by a power of two): the E8M0 byte
// (e = floor(log2 amax) - 2 from the fp32 exponent, clamped to [-127, 127]; 0 for a zero or
// subnormal amax) and 16 bytes of codes, element 2i in the low nibble, sign bits from the inputs.
__device__ __forceinline__ void code_mx_f32(const float (&v)[32], uint4& codes, uint32_t& byte) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int E = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  const int e = (E == 0) ? -127 : max(E - 129, -127);
  // 2^-e as two exact power-of-two factors (2^-e alone overflows fp32 for e = -127)
  const float inv1 = __uint_as_float(static_cast<uint32_t>(127 - (e >> 1)) << 23);
  const float inv2 = __uint_as_float(static_cast<uint32_t>(127 - (e - (e >> 1))) << 23);
  uint32_t packed[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float f[8];
    uint32_t sgn = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[i] = __fmul_rn(__fmul_rn(v[8 * q + i], inv1), inv2);
      sgn |= ((__float_as_uint(v[8 * q + i]) >> 31) << 3) << (4 * i);
    }
    packed[q] = e2m1x8(f) | sgn;
  }
  codes = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  byte = static_cast<uint32_t>(e + 127);
}

// One thread per 32-element block (4 x 16-byte loads in flight, one 16-byte code store).
// x: bf16 [M, K] with row stride ldx (elements).  codes: [M, K/2] bytes (row stride ldc),
// low nibble = even k.  Scales go to the plain [M, K/32] layout and/or the tiled layout.
// The first `nzero` ints of `zero_words` are cleared (scratch the consumer expects zeroed).
// deq_out (optional, [M, K] bf16) receives the exact value of every quantized element.
__global__ void __launch_bounds__(256) quant_mx_e8m0_b32_kernel(
    const __nv_bfloat16* __restrict__ x, int M, int K, int ldx, uint8_t* __restrict__ codes,
    int ldc, uint8_t* __restrict__ scales_plain, int lds, uint8_t* __restrict__ scales_tiled,
    int sf_atoms_per_row, int sf_tile_rows, int* __restrict__ zero_words, int nzero,
    __nv_bfloat16* __restrict__ deq_out = nullptr, int had = 0, int tail_from = -1,
    int tail_to = 0) {
  griddep_launch_dependents();   // a GEMM launched behind this grid may start streaming weights
  const long gtid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (zero_words != nullptr && gtid < nzero) zero_words[gtid] = 0;
  const int nblk = K >> 5;
  if (gtid >= static_cast<long>(M) * nblk) return;
  const int m = static_cast<int>(gtid / nblk);
  const int j = static_cast<int>(gtid - static_cast<long>(m) * nblk);
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * ldx) + j * 4;
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = __ldg(src + i);
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  uint32_t packed[4];
  int e;
  if (had) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    fwht32(v);
    uint4 c4;
    uint32_t byte;
    code_mx_f32(v, c4, byte);
    packed[0] = c4.x; packed[1] = c4.y; packed[2] = c4.z; packed[3] = c4.w;
    e = static_cast<int>(byte) - 127;
  } else {
    // amax over 32 bf16 magnitudes as 16-bit unsigned integers (order-preserving for finite values)
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) mx = __vmaxu2(mx, w[i] & 0x7FFF7FFFu);
    const uint32_t amax16 = max(mx & 0xFFFFu, mx >> 16);
    // floor(log2 amax) from the bf16 exponent field; zero or subnormal amax clamps to e = -127.
    const int E = static_cast<int>(amax16 >> 7);
    e = (E == 0) ? -127 : max(E - 129, -127);
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, normal
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float f[8];
      const uint32_t ww[4] = {w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(ww[i] << 16) * inv;
        f[2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u) * inv;
      }
      packed[q] = e2m1x8(f) | bf16x8_sign_nibbles(ww);
    }
  }
  const uint8_t b = static_cast<uint8_t>(e + 127);
  // PRQuant offline copy: blocks of the last channels [tail_from, K) are written a second time
  // at [tail_to, ...), so that the codes hold the augmented activation [Z~, Z~_tail]
  const int ncopy = (tail_from >= 0 && j * 32 >= tail_from) ? 2 : 1;
  for (int cpy = 0; cpy < ncopy; ++cpy) {
    const int jd = cpy == 0 ? j : (tail_to + j * 32 - tail_from) >> 5;
    *reinterpret_cast<uint4*>(codes + static_cast<size_t>(m) * ldc + jd * 16) =
        make_uint4(packed[0], packed[1], packed[2], packed[3]);
    if (scales_plain != nullptr) scales_plain[static_cast<size_t>(m) * lds + jd] = b;
    if (scales_tiled != nullptr) scales_tiled[sf_tiled_offset(m, jd, sf_atoms_per_row, sf_tile_rows)] = b;
  }
  if (deq_out != nullptr) {
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t c0 = (packed[i >> 2] >> (8 * (i & 3))) & 15u;
      const uint32_t c1 = (packed[i >> 2] >> (8 * (i & 3) + 4)) & 15u;
      const __nv_bfloat162 v = __floats2bfloat162_rn(ldexpf(e2m1_code_value(c0), e),
                                                     ldexpf(e2m1_code_value(c1), e));
      o[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    uint4* dst = reinterpret_cast<uint4*>(deq_out + static_cast<size_t>(m) * K + j * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
  }
}

// ------------------------------------------------------------------ E4M3-B16 + FP32 tensor scale
// MXCode, Table 1 row E4M3-B16-FP4: per 16 elements an E4M3 block scale and one FP32 tensor
// scale for the whole tensor.  Steps, each an IEEE fp32 operation in this order:
//   ts = amax_T / 2688 (1 if amax_T == 0);  s = E4M3_RNE_satfinite((amax_b / 6) / ts);
//   S = dec(s) * ts;  code = E2M1_RNE_satfinite(x / S)  (zero codes, sign kept, when S == 0).

// Largest |x| of a bf16 tensor as a bf16 bit pattern (16-bit magnitude), max-reduced into
// *amax16 (which the caller zeroes first).  n8 = number of 8-element (16-byte) groups.
__global__ void __launch_bounds__(256) absmax_bf16_kernel(const __nv_bfloat16* __restrict__ x,
                                                           long n8, unsigned* __restrict__ amax16) {
  uint32_t mx = 0;
  const uint4* src = reinterpret_cast<const uint4*>(x);
  for (long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(src + i);
    mx = __vmaxu2(mx, v.x & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, v.y & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, v.z & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, v.w & 0x7FFF7FFFu);
  }
  uint32_t m = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) b = max(b, red[w]);
    atomicMax(amax16, b);
  }
}

__device__ __forceinline__ float tensor_scale_from_amax16(uint32_t amax16) {
  const float amax = __uint_as_float(amax16 << 16);
  return amax == 0.f ? 1.f : __fdiv_rn(amax, 2688.0f);
}

// Value of a non-negative E4M3 byte (bias 7; subnormals m * 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return e == 0 ? static_cast<float>(m) * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// E4M3-B16 coding of one 16-element block held as 8 bf16x2 words (element 2i in the low half
// of w[i]) with tensor scale ts: its two packed code words (elements 0..7, 8..15) and its E4M3
// scale byte; the callers store them where their layouts want them.
__device__ __forceinline__ void quant_e4m3_code_block(const uint32_t (&w)[8], float ts,
                                                      uint32_t (&packed)[2], uint32_t& sb_out) {
  uint32_t mx = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) mx = __vmaxu2(mx, w[i] & 0x7FFF7FFFu);
  const float amax_b = __uint_as_float(max(mx & 0xFFFFu, mx >> 16) << 16);
  const float r = __fdiv_rn(__fdiv_rn(amax_b, 6.0f), ts);
  const uint32_t sb = static_cast<uint32_t>(__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3));
  const float S = __fmul_rn(e4m3_value(sb), ts);
  // Codes of the fp32 quotients q = RN(|x| / S), without a division per element: with
  // inv = RN(1/S) and r = RN(|x| * inv), r is within 2^-22 (relative) of q, so
  //   RN(r * (1 - 2^-21)) < q < RN(r * (1 + 2^-21))
  // (the constants are exact in fp32).  E2M1 round-to-nearest-even is monotone in q, so when the
  // codes of both bounds agree they are the code of q.  Otherwise -- a bound straddles a
  // rounding threshold, which almost never happens -- q is computed by the correctly rounded
  // division.  The bound needs S normal (so 1/S is finite); subnormal S takes the exact path.
  // Codes are formed from magnitudes and the sign of x is or-ed in (a negative x that rounds
  // to zero keeps code 0x8).
  const bool fast = S >= 0x1p-126f;
  const float inv = fast ? __frcp_rn(S) : 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t ww[4] = {w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]};
    float a[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[2 * i] = __uint_as_float((ww[i] << 16) & 0x7FFF0000u);
      a[2 * i + 1] = __uint_as_float(ww[i] & 0x7FFF0000u);
    }
    uint32_t code = 0;
    bool done = false;
    if (fast) {
      float lo[8], hi[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float r = __fmul_rn(a[i], inv);
        lo[i] = __fmul_rn(r, 0x1.fffffp-1f);   // 1 - 2^-21
        hi[i] = __fmul_rn(r, 0x1.00001p+0f);   // 1 + 2^-21
      }
      const uint32_t cl = e2m1x8(lo), ch = e2m1x8(hi);
      done = (cl == ch);
      code = cl;
    }
    if (!done) {
      float f[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = S == 0.f ? 0.f : __fdiv_rn(a[i], S);
      code = e2m1x8(f);
    }
    packed[h] = code | bf16x8_sign_nibbles(ww);
  }
  sb_out = sb;
}

// Quantize the 16-element block j of row m with tensor scale ts: codes [M, K/2] (row stride
// ldc), scales plain [M, K/16] and/or tiled (atoms of 64 K), from the block's 16 bf16 values
// already in registers.
__device__ __forceinline__ void quant_e4m3_regs(
    const uint32_t (&w)[8], int m, int j, float ts, uint8_t* __restrict__ codes, int ldc,
    uint8_t* __restrict__ scales_plain, int lds, uint8_t* __restrict__ scales_tiled,
    int sf_atoms_per_row, int sf_tile_rows) {
  uint32_t packed[2], sb;
  quant_e4m3_code_block(w, ts, packed, sb);
  *reinterpret_cast<uint2*>(codes + static_cast<size_t>(m) * ldc + j * 8) =
      make_uint2(packed[0], packed[1]);
  if (scales_plain != nullptr) scales_plain[static_cast<size_t>(m) * lds + j] = static_cast<uint8_t>(sb);
  if (scales_tiled != nullptr)
    scales_tiled[sf_tiled_offset(m, j, sf_atoms_per_row, sf_tile_rows)] = static_cast<uint8_t>(sb);
}

__device__ __forceinline__ void quant_e4m3_block(
    const __nv_bfloat16* __restrict__ x, int m, int j, int ldx, float ts, uint8_t* __restrict__ codes,
    int ldc, uint8_t* __restrict__ scales_plain, int lds, uint8_t* __restrict__ scales_tiled,
    int sf_atoms_per_row, int sf_tile_rows) {
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * ldx) + j * 2;
  const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  quant_e4m3_regs(w, m, j, ts, codes, ldc, scales_plain, lds, scales_tiled, sf_atoms_per_row, sf_tile_rows);
}

// One thread per 16-element block, tensor scale from the amax that absmax_bf16_kernel reduced.
// Thread 0 stores ts to *ts_out when ts_out is not null.
__global__ void __launch_bounds__(256) quant_e4m3_b16_kernel(
    const __nv_bfloat16* __restrict__ x, int M, int K, int ldx, const unsigned* __restrict__ amax16,
    float* __restrict__ ts_out, uint8_t* __restrict__ codes, int ldc,
    uint8_t* __restrict__ scales_plain, int lds, uint8_t* __restrict__ scales_tiled,
    int sf_atoms_per_row, int sf_tile_rows) {
  griddep_launch_dependents();   // a GEMM launched behind this grid may start streaming weights
  const long gtid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const float ts = tensor_scale_from_amax16(*amax16);
  if (gtid == 0 && ts_out != nullptr) *ts_out = ts;
  const int nblk = K >> 4;
  if (gtid >= static_cast<long>(M) * nblk) return;
  const int m = static_cast<int>(gtid / nblk);
  const int j = static_cast<int>(gtid - static_cast<long>(m) * nblk);
  quant_e4m3_block(x, m, j, ldx, ts, codes, ldc, scales_plain, lds, scales_tiled, sf_atoms_per_row, sf_tile_rows);
}

// Small tensors (decode): one thread-block cluster does the whole job in one launch.  Each thread
// loads its (at most kE4m3RegBlocks) 16-element blocks once and keeps them in registers; every CTA
// pushes its maximum into a slot of every CTA's shared memory (distributed shared memory), one
// cluster barrier later each CTA has all maxima locally, and the blocks are quantized from
// registers.  Launched with programmatic stream serialization: it first lets the GEMM behind it
// launch (that grid streams weights until its own griddepcontrol.wait, which returns only after
// this grid completes), then waits for the grid before it (which may produce x).  The amax bit
// pattern goes to *amax_out and ts to *ts_out (either may be null); the first nzero ints of
// zero_words are cleared.
constexpr int kE4m3RegBlocks = 3;
constexpr int kE4m3ClusterThreads = 1024;
__global__ void __launch_bounds__(kE4m3ClusterThreads) quant_e4m3_b16_cluster_kernel(
    const __nv_bfloat16* __restrict__ x, int M, int K, int ldx, unsigned* __restrict__ amax_out,
    float* __restrict__ ts_out, uint8_t* __restrict__ codes, int ldc,
    uint8_t* __restrict__ scales_plain, int lds, uint8_t* __restrict__ scales_tiled,
    int sf_atoms_per_row, int sf_tile_rows, int* __restrict__ zero_words, int nzero) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ uint32_t red[kE4m3ClusterThreads / 32];
  __shared__ uint32_t s_slot[16];   // CTA maxima of the cluster's ranks
  const int ncta = static_cast<int>(gridDim.x);   // the grid is one cluster (<= 16 CTAs)
  const long tid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long nthr = static_cast<long>(ncta) * blockDim.x;
  const int nblk = K >> 4;
  const long total = static_cast<long>(M) * nblk;
  uint32_t w[kE4m3RegBlocks][8];
  uint32_t mx = 0;
#pragma unroll
  for (int k = 0; k < kE4m3RegBlocks; ++k) {
    const long b = tid + k * nthr;
    if (b < total) {
      const int m = static_cast<int>(b / nblk);
      const int j = static_cast<int>(b - static_cast<long>(m) * nblk);
      const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * ldx) + j * 2;
      const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
      w[k][0] = v0.x; w[k][1] = v0.y; w[k][2] = v0.z; w[k][3] = v0.w;
      w[k][4] = v1.x; w[k][5] = v1.y; w[k][6] = v1.z; w[k][7] = v1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = __vmaxu2(mx, w[k][i] & 0x7FFF7FFFu);
    }
  }
  uint32_t m16 = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m16 = max(m16, __shfl_xor_sync(0xFFFFFFFFu, m16, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m16;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    if (static_cast<int>(threadIdx.x) < ncta)   // lane t pushes this CTA's maximum to rank t
      st_shared_cluster_u32(map_shared_rank(smem_u32(&s_slot[blockIdx.x]), threadIdx.x), v);
  }
  cluster_sync_all();
  uint32_t amax16 = 0;
  for (int r = 0; r < ncta; ++r) amax16 = max(amax16, s_slot[r]);
  const float ts = tensor_scale_from_amax16(amax16);
  if (tid == 0) {
    if (amax_out != nullptr) *amax_out = amax16;
    if (ts_out != nullptr) *ts_out = ts;
  }
  if (zero_words != nullptr)
    for (long i = tid; i < nzero; i += nthr) zero_words[i] = 0;
#pragma unroll
  for (int k = 0; k < kE4m3RegBlocks; ++k) {
    const long b = tid + k * nthr;
    if (b < total) {
      const int m = static_cast<int>(b / nblk);
      const int j = static_cast<int>(b - static_cast<long>(m) * nblk);
      quant_e4m3_regs(w[k], m, j, ts, codes, ldc, scales_plain, lds, scales_tiled, sf_atoms_per_row, sf_tile_rows);
    }
  }
}

// Mid-size tensors (a few decode tokens up to ~1.8 M elements): one grid of small CTAs, at most one
// per SM, so that all of them are resident at once, also beside a running GEMM CTA.  Each thread
// keeps its (at most kE4m3RegBlocks) 16-element blocks in registers.  The tensor amax is agreed on
// through the workspace block `sync`: word 0 a launch counter, bytes 8..15 a result word, then one
// 64-bit slot per CTA.  Every CTA reads the counter c once and publishes its maximum in its slot,
// tagged with c + 1 (release).  CTA 0 waits (bounded) until every slot carries the tag (acquire),
// stores the tagged maximum of all of them in the result word and advances the counter; the other
// CTAs wait for the tagged result (one word, so the polling does not pile onto the slots' cache
// lines).  No word needs clearing between launches; a stale word would have to repeat a 48-bit tag
// to be taken for a fresh one.  Launched with programmatic stream serialization like the cluster
// kernel.  On a timeout the error word is set and no codes are written, and each CTA whose wait
// expired advances the counter by two, so the next launch's tag matches no word left behind.
constexpr int kE4m3GridThreads = 256;
constexpr int kE4m3GridMaxCtas = 256;   // CTA 0 polls one slot per thread
constexpr int kE4m3SyncBytes = 16 + 8 * kE4m3GridMaxCtas;

__device__ __forceinline__ unsigned long long e4m3_grid_tag(uint32_t c) {
  return (static_cast<unsigned long long>(c) << 32) |
         (static_cast<unsigned long long>((c * 0x9E37u + 0x5A3Cu) & 0xFFFFu) << 16);
}

// Bounded wait until *p carries `tag` in its upper 48 bits; returns the word (0 on a timeout).
__device__ __forceinline__ unsigned long long wait_tagged_u64(const unsigned long long* p,
                                                              unsigned long long tag, bool& ok) {
  unsigned long long s = ld_acquire_gpu_u64(p);
  if ((s & ~0xFFFFull) == tag) return s;
  const uint64_t t0 = globaltimer_ns(), limit = wait_limit_ns();
  while (true) {
    __nanosleep(64);
    s = ld_acquire_gpu_u64(p);
    if ((s & ~0xFFFFull) == tag) return s;
    if (globaltimer_ns() - t0 > limit) {
      record_error(DEV_TIMEOUT, 30);
      ok = false;
      return 0;
    }
  }
}

__global__ void __launch_bounds__(kE4m3GridThreads) quant_e4m3_b16_grid_kernel(
    const __nv_bfloat16* __restrict__ x, int M, int K, int ldx, unsigned* __restrict__ amax_out,
    float* __restrict__ ts_out, uint8_t* __restrict__ codes, int ldc,
    uint8_t* __restrict__ scales_plain, int lds, uint8_t* __restrict__ scales_tiled,
    int sf_atoms_per_row, int sf_tile_rows, int* __restrict__ zero_words, int nzero, uint32_t* __restrict__ sync) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ uint32_t red[kE4m3GridThreads / 32];
  __shared__ uint32_t s_count, s_amax;
  __shared__ int s_ok;
  unsigned long long* result = reinterpret_cast<unsigned long long*>(sync + 2);
  unsigned long long* slots = result + 1;
  if (threadIdx.x == 0) s_count = *reinterpret_cast<volatile uint32_t*>(sync) + 1u;
  const long tid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long nthr = static_cast<long>(gridDim.x) * blockDim.x;
  const int nblk = K >> 4;
  const long total = static_cast<long>(M) * nblk;
  uint32_t w[kE4m3RegBlocks][8];
  uint32_t mx = 0;
#pragma unroll
  for (int k = 0; k < kE4m3RegBlocks; ++k) {
    const long b = tid + k * nthr;
    if (b < total) {
      const int m = static_cast<int>(b / nblk);
      const int j = static_cast<int>(b - static_cast<long>(m) * nblk);
      const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * ldx) + j * 2;
      const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
      w[k][0] = v0.x; w[k][1] = v0.y; w[k][2] = v0.z; w[k][3] = v0.w;
      w[k][4] = v1.x; w[k][5] = v1.y; w[k][6] = v1.z; w[k][7] = v1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = __vmaxu2(mx, w[k][i] & 0x7FFF7FFFu);
    }
  }
  if (zero_words != nullptr)
    for (long i = tid; i < nzero; i += nthr) zero_words[i] = 0;
  uint32_t m16 = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m16 = max(m16, __shfl_xor_sync(0xFFFFFFFFu, m16, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m16;
  __syncthreads();   // also publishes s_count
  const uint32_t cnt = s_count;
  const unsigned long long tag = e4m3_grid_tag(cnt);
  if (threadIdx.x == 0 && !withheld(blockIdx.x)) {
    uint32_t v = 0;
    for (int i = 0; i < kE4m3GridThreads / 32; ++i) v = max(v, red[i]);
    st_release_gpu_u64(&slots[blockIdx.x], tag | v);
  }
  bool ok = true;
  if (blockIdx.x == 0) {
    uint32_t a16 = 0;
    if (threadIdx.x < gridDim.x)
      a16 = static_cast<uint32_t>(wait_tagged_u64(&slots[threadIdx.x], tag, ok) & 0xFFFFull);
    __syncthreads();   // red[] is reused
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a16 = max(a16, __shfl_xor_sync(0xFFFFFFFFu, a16, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a16;
    ok = __syncthreads_and(ok);
    if (threadIdx.x == 0) {
      uint32_t v = 0;
      for (int i = 0; i < kE4m3GridThreads / 32; ++i) v = max(v, red[i]);
      s_amax = v;
      if (ok) {
        st_release_gpu_u64(result, tag | v);
        atomicAdd(sync, 1u);   // every CTA has read the counter (its slot carries the tag)
      }
    }
  } else if (threadIdx.x == 0) {
    s_ok = 1;
    s_amax = static_cast<uint32_t>(wait_tagged_u64(result, tag, ok) & 0xFFFFull);
    s_ok = ok;
  }
  __syncthreads();
  if (blockIdx.x != 0) ok = s_ok != 0;
  if (!ok) {
    // A CTA whose wait expired moves the counter on by two: one that read it late (value v,
    // after CTA 0 gave up) tagged its slot v + 1 and leaves the counter at v + 2 or more, so no
    // word of this launch can match the next launch's tag; the workspace needs no clearing.
    if (threadIdx.x == 0) atomicAdd(sync, 2u);
    return;
  }
  const uint32_t amax16 = s_amax;
  const float ts = tensor_scale_from_amax16(amax16);
  if (tid == 0) {
    if (amax_out != nullptr) *amax_out = amax16;
    if (ts_out != nullptr) *ts_out = ts;
  }
#pragma unroll
  for (int k = 0; k < kE4m3RegBlocks; ++k) {
    const long b = tid + k * nthr;
    if (b < total) {
      const int m = static_cast<int>(b / nblk);
      const int j = static_cast<int>(b - static_cast<long>(m) * nblk);
      quant_e4m3_regs(w[k], m, j, ts, codes, ldc, scales_plain, lds, scales_tiled, sf_atoms_per_row, sf_tile_rows);
    }
  }
}

// Replace the amax bit pattern stored in *slot by the tensor scale it implies (single thread).
__global__ void amax_to_tensor_scale_kernel(unsigned* slot) {
  const float ts = tensor_scale_from_amax16(*slot);
  *reinterpret_cast<float*>(slot) = ts;
}

}  // namespace ql
