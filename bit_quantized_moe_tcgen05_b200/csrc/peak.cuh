// Tensor-pipe throughput microbenchmark for the roofline denominators (sm_100a).
//
// Each CTA (one per SM) keeps one A tile (128 rows) and one B tile (N rows) resident in shared
// memory, 256 bytes deep along K, and has one thread issue back-to-back tcgen05.mma instructions
// into a single TMEM accumulator, which is what the inner loop of a GEMM does once its operands
// have landed.  No operand is re-loaded, so the time is the tensor pipe's alone: an upper bound
// for any GEMM of the same instruction kind.  Kinds:
//   0  kind::mxf4.block_scale.block32      (E2M1 x E2M1, E8M0 scales per 32; 64 K per MMA)
//   1  kind::mxf4nvf4.block_scale.block16  (E2M1 x E2M1, UE4M3 scales per 16; 64 K per MMA)
//   2  kind::i8                            (s8 x s8 -> s32; 32 K per MMA)
//   3  kind::f16 with bf16 operands        (16 K per MMA) -- the same loop on the pipe whose
//                                            cuBLAS throughput is measured independently, as a
//                                            check of the method
// The operand bytes are a fixed pattern of finite values (results are not read back).
#pragma once
#include "ptx.cuh"

namespace ql {

template <int KIND, int N>
struct PeakCfg {
  static constexpr int kABytes = 128 * 128;      // 128 rows x 128 B (one 128-byte swizzle atom wide)
  static constexpr int kBBytes = N * 128;
  static constexpr int kSfBytes = 2 * 512;       // two scale atoms (A and B), block-scaled kinds
  static constexpr int kSmem = kABytes + kBBytes + kSfBytes + 1024;
  // MMAs per 128-byte K slice: fp4 64 K x 4 bits = 32 B; i8 32 K = 32 B; bf16 16 K = 32 B
  static constexpr int kMmaPerTile = 4;
  static constexpr int kKPerMma = KIND <= 1 ? 64 : KIND == 2 ? 32 : 16;
  static constexpr double kFlopsPerMma = 2.0 * 128 * N * kKPerMma;
};

template <int KIND, int N>
__global__ void __launch_bounds__(128, 1) tensor_peak_kernel(int iters) {
  using Cfg = PeakCfg<KIND, N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + Cfg::kABytes;
  uint8_t* sSf = sB + Cfg::kBBytes;
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;
  // finite operand pattern: 0x22 = two E2M1 codes of 1.0 / the int8 34 / half of the bf16 1.0625
  // pair 0x3F88 when read with 0x3F; scales: E8M0 127 (1.0), UE4M3 0x38 (1.0)
  for (int i = threadIdx.x; i < (Cfg::kABytes + Cfg::kBBytes) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sA)[i] = KIND == 3 ? 0x3F883F88u : 0x22222222u;
  for (int i = threadIdx.x; i < Cfg::kSfBytes / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sSf)[i] = KIND == 0 ? 0x7F7F7F7Fu : 0x38383838u;
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) {
    const uint32_t tsfa = tmem + 256, tsfb = tmem + 260;
    if (KIND <= 1) {
      tc_cp_32x128b_warpx4(tsfa, make_sdesc(smem_u32(sSf), 0, 128, kLayoutNone));
      tc_cp_32x128b_warpx4(tsfb, make_sdesc(smem_u32(sSf + 512), 0, 128, kLayoutNone));
    }
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    uint32_t idesc = KIND <= 1 ? idesc_fp4_block(N, KIND == 0) : KIND == 2 ? idesc_s8(N) : idesc_bf16(N);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < Cfg::kMmaPerTile; ++kk) {
        const uint64_t ad = make_sdesc(a0 + kk * 32, 16, 1024, kLayoutSW128);
        const uint64_t bd = make_sdesc(b0 + kk * 32, 16, 1024, kLayoutSW128);
        const uint32_t acc = (it | kk) ? 1u : 0u;
        if constexpr (KIND == 0)
          mma_mxf4_block32(tmem, ad, bd, idesc, tsfa, tsfb, acc);
        else if constexpr (KIND == 1)
          mma_nvf4_block16(tmem, ad, bd, idesc, tsfa, tsfb, acc);
        else if constexpr (KIND == 2)
          mma_i8(tmem, ad, bd, idesc, acc);
        else
          mma_f16(tmem, ad, bd, idesc, acc);
      }
    }
    tc_commit(&done);
  }
  __syncwarp();
  // every MMA has completed once the commit arrives; bounded wait (records the error word)
  if (warp == 0) mbar_wait(&done, 0, 40, 4000000000ull);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace ql
