// INT4 dense base + block-sparse INT4 residual, fused in one tcgen05 GEMM (sm_100a).
//
// MosaicQuant, "ZipperEngine": the sparse compensation and the output merge run inside the dense
// GEMM.  Here every 128-row weight tile owns a list of K stages: the 64 base groups of 128 input
// channels, then one stage per input group in which any of the tile's 16-row blocks carries a
// residual block (rows without one are zero).  A stage is one contiguous block in HBM: 128 rows of
// packed INT4 codes (64 B each) and 128 fp32 row scales (the base scale, or the residual scale).
//
//   y[m, n] = sum_stages  s_row[n] * sx[m, g] * I[m, n],   I = exact int32 dot product over the group
//
// Warps: 0 producer (1-D bulk copies of the weight block and the activation group's scales, TMA
// tile of the int8 activation), 1 MMA (kind::i8 into one of two TMEM int32 accumulators),
// 2..5 fold (read the group's int32 result, multiply by the two scales, accumulate in fp32
// registers; then the epilogue), 6..9 decode (INT4 nibbles -> int8 operand tile, 128-byte swizzle).
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant_act.cuh"

namespace ql {

// Most K-splits of one INT4 output tile; the splits form one thread-block cluster.
constexpr int kInt4MaxClusterSplits = 4;

// ------------------------------------------------------------------ INT4 activation quantizer
// One warp per (token, 128-group): s = amax / 7 (fp32), q = clamp(rint(x / s), -7, 7) (fp32
// divide, ties to even), q = 0 when s == 0.  Outputs (each optional): int8 codes [M, K] (row
// stride K), packed int4 [M, K/2], scales [M, K/128], transposed scales [K/128][ldt].
__global__ void __launch_bounds__(256) quant_int4_g128_kernel(
    const __nv_bfloat16* __restrict__ x, int M, int K, int8_t* __restrict__ q8,
    uint8_t* __restrict__ q4, float* __restrict__ scales, float* __restrict__ scales_t, int ldt) {
  const long wid = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int G = K >> 7;
  if (wid >= static_cast<long>(M) * G) return;
  const int m = static_cast<int>(wid / G), g = static_cast<int>(wid % G);
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(x + static_cast<size_t>(m) * K + g * 128) + lane);
  const float f[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                      __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u)};
  float amax = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const float s = __fdiv_rn(amax, 7.0f);
  int q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float r = s == 0.f ? 0.f : rintf(__fdiv_rn(f[i], s));
    q[i] = static_cast<int>(fminf(7.f, fmaxf(-7.f, r)));
  }
  if (q8 != nullptr) {
    const uint32_t w = (q[0] & 255) | ((q[1] & 255) << 8) | ((q[2] & 255) << 16) | ((q[3] & 255u) << 24);
    *reinterpret_cast<uint32_t*>(q8 + static_cast<size_t>(m) * K + g * 128 + lane * 4) = w;
  }
  if (q4 != nullptr) {
    const uint32_t w = (q[0] & 15) | ((q[1] & 15) << 4) | ((q[2] & 15) << 8) | ((q[3] & 15) << 12);
    *reinterpret_cast<uint16_t*>(q4 + static_cast<size_t>(m) * (K / 2) + g * 64 + lane * 2) =
        static_cast<uint16_t>(w);
  }
  if (lane == 0) {
    if (scales != nullptr) scales[static_cast<size_t>(m) * G + g] = s;
    if (scales_t != nullptr) scales_t[static_cast<size_t>(g) * ldt + m] = s;
  }
}

// ------------------------------------------------------------------ fused GEMM
struct Int4GemmArgs {
  int M, N;
  const uint8_t* wblocks;        // stage blocks: [128][64 B] codes then [128] fp32 row scales
  const int* stage_start;        // [N/128 + 1] first stage of each weight tile
  const int* stage_group;        // [stages] activation group of each stage
  const float* sx_t;             // [K/128][ldt] activation scales, transposed
  int ldt;
  int stages_per_split;          // gridDim.z = splits (a cluster along z)
  __nv_bfloat16* y;
  float* y32;
};

constexpr int kInt4WBlock = 128 * 64 + 128 * 4;   // 8704 B

template <int BN>
struct Int4Cfg {
  // warps: 0 producer, 1 MMA, then kFoldWarps fold/epilogue warps, then 4 decode warps
  static constexpr int kFoldWarps = BN >= 128 ? 8 : 4;
  static constexpr int kCols = BN * 4 / kFoldWarps;   // accumulator columns per fold thread
  static constexpr int kDecWarps = 4;
  static constexpr int kThreads = (2 + kFoldWarps + kDecWarps) * 32;
  static constexpr int kRawBytes = kInt4WBlock;
  static constexpr int kABytes = 128 * 128;        // int8 tile, 128 rows x 128 B
  static constexpr int kBBytes = BN * 128;
  static constexpr int kSxBytes = BN * 4 < 16 ? 16 : BN * 4;
  static constexpr int kStageBytes = ((kRawBytes + kABytes + kBBytes + kSxBytes) + 1023) / 1024 * 1024;
  static constexpr int kStagesRaw = (200 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 512;
  static_assert(BN * 128 * 4 <= kStages * kStageBytes, "output staging must fit the ring");
  static_assert(kCols % 8 == 0, "fold columns come in tcgen05.ld groups of 8");
};

// Packed fp32 pair arithmetic (sm_100 f32x2 instructions): d = a * b + c, d = a + b, d = a * b,
// each element rounded to nearest even exactly as the scalar instruction would.
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// Exact float of an int32 x with |x| < 2^22: in [2^23, 2^24) the float grid is the integers, so
// the bit pattern of 1.5 * 2^23 plus x is the float 1.5 * 2^23 + x; the subtraction is exact.
// (Starting the TMEM accumulators at that bit pattern, re-written by the fold after each read,
// would save the integer adds; the extra TMEM stores measured far slower.)
__device__ __forceinline__ float2 small_ints_to_float2(uint32_t x0, uint32_t x1) {
  return f2_add(make_float2(__uint_as_float(x0 + 0x4B400000u), __uint_as_float(x1 + 0x4B400000u)),
                make_float2(-12582912.0f, -12582912.0f));
}
// Sign-extend the eight 4-bit two's-complement fields of w to bytes: lo gets the low nibble of each
// byte, hi the high nibble. A field with bit 3 set gains 0xF0 (8 * 30 = 240 stays inside its byte).
__device__ __forceinline__ void int4x8_to_int8(uint32_t w, uint32_t& lo, uint32_t& hi) {
  lo = (w & 0x0F0F0F0Fu) | ((w & 0x08080808u) * 30u);
  const uint32_t w4 = w >> 4;
  hi = (w4 & 0x0F0F0F0Fu) | ((w4 & 0x08080808u) * 30u);
}

template <int BN>
__global__ void __launch_bounds__(Int4Cfg<BN>::kThreads, 1)
    int4_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
                     const __grid_constant__ CUtensorMap tm_y32, const Int4GemmArgs a) {
  using Cfg = Int4Cfg<BN>;
  constexpr int S = Cfg::kStages;
  constexpr int kFoldThreads = Cfg::kFoldWarps * 32;
  extern __shared__ uint8_t smem_raw[];
  // 1 KB aligned by offsetting the shared array itself, so that every pointer derived from it
  // stays a shared-space pointer (plain ld/st.shared, not generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  // stage st: [A int8 tile 16 KB][B tile][raw weight block][sx]  (A and B 1024-aligned)
  auto sA = [&](int st) { return smem + st * Cfg::kStageBytes; };
  auto sB = [&](int st) { return smem + st * Cfg::kStageBytes + Cfg::kABytes; };
  auto sRaw = [&](int st) { return smem + st * Cfg::kStageBytes + Cfg::kABytes + Cfg::kBBytes; };
  auto sSx = [&](int st) {
    return reinterpret_cast<float*>(smem + st * Cfg::kStageBytes + Cfg::kABytes + Cfg::kBBytes + Cfg::kRawBytes);
  };
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * Cfg::kStageBytes);
  uint64_t* empty = full + S;
  uint64_t* decd = empty + S;
  uint64_t* accf = decd + S;      // [2]
  uint64_t* acce = accf + 2;      // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, n0 = tile * 128, m0 = blockIdx.y * BN;
  const int st0 = a.stage_start[tile], st_n = a.stage_start[tile + 1] - st0;
  const int s_begin = blockIdx.z * a.stages_per_split;
  const int s_end = min(st_n, s_begin + a.stages_per_split);
  const int nst = max(0, s_end - s_begin);
  const bool fold_warp = warp >= 2 && warp < 2 + Cfg::kFoldWarps;
  const int fthread = threadIdx.x - 64;                       // 0.. fold threads - 1
  const int q = warp & 3;                                     // TMEM lane quadrant of a fold warp
  const int row = q * 32 + lane;                              // weight row of a fold thread
  const int col0 = (fthread / 128) * Cfg::kCols;              // its accumulator columns

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);     // MMA commit + fold release
      mbar_init(&decd[s], Cfg::kDecWarps * 32);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tm_x);
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tfold = tmem + (static_cast<uint32_t>(q * 32) << 16) + col0;   // a fold thread's lane and columns

  bool ok = true;
  float2 acc[Cfg::kCols / 2];
#pragma unroll
  for (int c = 0; c < Cfg::kCols / 2; ++c) acc[c] = make_float2(0.f, 0.f);

  if (warp == 0) {
    if (lane == 0) {
      for (int j = 0; j < nst && ok; ++j) {
        const int st = j % S;
        const uint32_t ph = (j / S) & 1;
        if (!mbar_wait(&empty[st], ph ^ 1, 21)) { ok = false; break; }
        const int gs = st0 + s_begin + j;
        const int g = a.stage_group[gs];
        mbar_arrive_expect_tx(&full[st], Cfg::kRawBytes + Cfg::kBBytes + BN * 4);
        bulk_load(sRaw(st), a.wblocks + static_cast<size_t>(gs) * kInt4WBlock, Cfg::kRawBytes, &full[st]);
        tma_load_2d(sB(st), &tm_x, &full[st], g * 128, m0);
        bulk_load(sSx(st), a.sx_t + static_cast<size_t>(g) * a.ldt + m0, BN * 4, &full[st]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_s8(BN);
      for (int j = 0; j < nst && ok; ++j) {
        const int st = j % S, b = j & 1;
        const uint32_t ph = (j / S) & 1;
        if (!mbar_wait(&full[st], ph, 22) || !mbar_wait(&decd[st], ph, 23) ||
            !mbar_wait(&acce[b], ((j >> 1) & 1) ^ 1, 24)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ab = smem_u32(sA(st)), bb = smem_u32(sB(st));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_i8(tmem + b * BN, make_sdesc(ab + kk * 32, 16, 1024, kLayoutSW128),
                 make_sdesc(bb + kk * 32, 16, 1024, kLayoutSW128), idesc, kk > 0 ? 1u : 0u);
        tc_commit(&empty[st]);
        tc_commit(&accf[b]);
      }
    }
  } else if (!fold_warp) {
    // ---------------- decode: packed INT4 -> int8, 128-byte swizzled K-major tile
    const int t = threadIdx.x - (2 + Cfg::kFoldWarps) * 32;
    for (int j = 0; j < nst && ok; ++j) {
      const int st = j % S;
      const uint32_t ph = (j / S) & 1;
      if (!mbar_wait(&full[st], ph, 25)) { ok = false; break; }
      const uint8_t* raw = sRaw(st);
      uint8_t* at = sA(st);
#pragma unroll 4
      for (int i = 0; i < 8; ++i) {
        const int c = t + 128 * i;                 // 16-byte output chunk: row r, chunk kc
        const int r = c >> 3, kc = c & 7;
        const uint2 pw = *reinterpret_cast<const uint2*>(raw + r * 64 + kc * 8);   // 16 nibbles
        uint32_t o[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t lo, hi;
          int4x8_to_int8(h ? pw.y : pw.x, lo, hi);
          o[2 * h] = __byte_perm(lo, hi, 0x5140);
          o[2 * h + 1] = __byte_perm(lo, hi, 0x7362);
        }
        *reinterpret_cast<uint4*>(at + r * 128 + ((kc ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&decd[st]);
    }
  } else {
    // ---------------- fold: acc += I * (s_w * s_x) per 128-input group, on packed fp32 pairs.
    // Fold warps own TMEM lane quadrant warp % 4 (weight rows) and a run of kCols columns.
    // The loop count is the same for all fold threads (named barrier inside); a thread whose wait
    // expired skips the work but keeps taking the barriers.
    for (int j = 0; j < nst; ++j) {
      const int st = j % S, b = j & 1;
      if (ok) ok = mbar_wait(&accf[b], (j >> 1) & 1, 26);
      tc_fence_after();
      if (ok) {
        const float rs = reinterpret_cast<const float*>(sRaw(st) + 128 * 64)[row];
        const float2 rs2 = make_float2(rs, rs);
        const float* sx = sSx(st) + col0;
        // the accumulator loads of up to 32 columns in flight at once, then one wait (a wait per
        // 8 columns serialised the TMEM latency eight times per stage)
        constexpr int kBatch = Cfg::kCols < 32 ? Cfg::kCols : 32;
#pragma unroll
        for (int c0 = 0; c0 < Cfg::kCols; c0 += kBatch) {
          uint32_t r[kBatch];
#pragma unroll
          for (int c = 0; c < kBatch; c += 8)
            tmem_ld8(tfold + b * BN + c0 + c, *reinterpret_cast<uint32_t(*)[8]>(r + c));
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < kBatch; c += 8) {
            const float4 s0 = *reinterpret_cast<const float4*>(sx + c0 + c);
            const float4 s1 = *reinterpret_cast<const float4*>(sx + c0 + c + 4);
            const float2 w0 = f2_mul(rs2, make_float2(s0.x, s0.y)), w1 = f2_mul(rs2, make_float2(s0.z, s0.w));
            const float2 w2 = f2_mul(rs2, make_float2(s1.x, s1.y)), w3 = f2_mul(rs2, make_float2(s1.z, s1.w));
            const int ca = (c0 + c) / 2;
            acc[ca + 0] = f2_fma(small_ints_to_float2(r[c + 0], r[c + 1]), w0, acc[ca + 0]);
            acc[ca + 1] = f2_fma(small_ints_to_float2(r[c + 2], r[c + 3]), w1, acc[ca + 1]);
            acc[ca + 2] = f2_fma(small_ints_to_float2(r[c + 4], r[c + 5]), w2, acc[ca + 2]);
            acc[ca + 3] = f2_fma(small_ints_to_float2(r[c + 6], r[c + 7]), w3, acc[ca + 3]);
          }
        }
      }
      tc_fence_before();
      named_bar_sync(2, kFoldThreads);
      if (fthread == 0) {
        mbar_arrive(&acce[b]);
        mbar_arrive(&empty[st]);
      }
    }
  }

  // ---------------- epilogue (fold warps): one tile, or a cluster of K-splits
  const int splits = gridDim.z;
  if (fold_warp) {
    named_bar_sync(2, kFoldThreads);   // every fold thread is past the ring
    if (splits == 1) {
      __nv_bfloat16* ybuf = reinterpret_cast<__nv_bfloat16*>(smem);
#pragma unroll
      for (int c = 0; c < Cfg::kCols / 2; ++c) {
        ybuf[(col0 + 2 * c) * 128 + row] = __float2bfloat16_rn(acc[c].x);
        ybuf[(col0 + 2 * c + 1) * 128 + row] = __float2bfloat16_rn(acc[c].y);
      }
      fence_proxy_async_smem();
      named_bar_sync(2, kFoldThreads);
      if (fthread == 0 && ok) {
        tma_store_2d(&tm_y, ybuf, n0, m0);
        bulk_commit_group();
        bulk_wait_group_read0();
      }
      if (a.y32 != nullptr) {
        named_bar_sync(2, kFoldThreads);
        float* y32buf = reinterpret_cast<float*>(smem);
#pragma unroll
        for (int c = 0; c < Cfg::kCols / 2; ++c) {
          y32buf[(col0 + 2 * c) * 128 + row] = acc[c].x;
          y32buf[(col0 + 2 * c + 1) * 128 + row] = acc[c].y;
        }
        fence_proxy_async_smem();
        named_bar_sync(2, kFoldThreads);
        if (fthread == 0 && ok) {
          tma_store_2d(&tm_y32, y32buf, n0, m0);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
      }
    } else {
      float* part = reinterpret_cast<float*>(smem);
#pragma unroll
      for (int c = 0; c < Cfg::kCols / 2; ++c) {
        part[(col0 + 2 * c) * 128 + row] = acc[c].x;
        part[(col0 + 2 * c + 1) * 128 + row] = acc[c].y;
      }
    }
  }
  __syncwarp();
  cluster_sync_all();
  if (splits > 1 && warp >= 2 && warp < 6) {
    const int qq = warp & 3;
    const int n = n0 + qq * 32 + lane;
    const int rank = static_cast<int>(cluster_ctarank());
    const int mcount = min(BN, a.M - m0);
    const uint32_t base = smem_u32(smem) + (qq * 32 + lane) * 4;
    for (int c = rank * 8; c < mcount; c += splits * 8) {
      float v[kInt4MaxClusterSplits][8];
#pragma unroll
      for (int r = 0; r < kInt4MaxClusterSplits; ++r)
        if (r < splits) {
          const uint32_t remote = map_shared_rank(base + c * 512, r);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[r][e] = ld_shared_cluster_f32(remote + e * 512);
        }
      if (n < a.N) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float sacc = 0.f;
#pragma unroll
          for (int r = 0; r < kInt4MaxClusterSplits; ++r)
            if (r < splits) sacc += v[r][e];
          if (c + e < mcount) {
            const size_t o = static_cast<size_t>(m0 + c + e) * a.N + n;
            a.y[o] = __float2bfloat16_rn(sacc);
            if (a.y32 != nullptr) a.y32[o] = sacc;
          }
        }
      }
    }
  }
  cluster_sync_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace ql
