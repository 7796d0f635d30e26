// Routed MoE FFN with cluster-codebook experts on sm_100a.
//
// CodeQuant ("Unified Clustering and Quantization ..."), Figure 1 Stage 4 and Figure 4: the
// deployed kernel rebuilds each weight tile from a lookup table held in SM shared memory.  Here a
// weight row owns 16 bf16 centroids and each weight is a 4-bit index into them; decoder warps turn
// a stage's indices into a bf16 operand tile in the MMA's 128-byte-swizzled layout, and the
// tensor cores run tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in TMEM).  Activations are MXFP4
// (E8M0-B32), dequantized exactly to bf16 for the MMA.
//
// Kernels, in launch order:
//   moe_topk_kernel        top-k of the router logits per token (ties to the lower expert id),
//                          softmax gate weights, per-expert counts
//   moe_scatter_kernel     one CTA per expert: offsets and the expert's routed entries
//                          (f = t*k + s) in ascending (t, s) order -- deterministic
//   quant_mx_e8m0_b32_kernel (quant_act.cuh) with a bf16 dequantized copy of x
//   moe_gemm_kernel<GATEUP> gate/up: B rows gathered per entry by TMA tile::gather4; epilogue
//                          h = silu(g) * u, MXFP4 requantization of h per 32 features, and the
//                          exact bf16 value of the quantized h for the down projection
//   moe_gemm_kernel<DOWN>  down: B = the expert's contiguous h rows; epilogue writes
//                          gate * y into a per-slot fp32 buffer
//   moe_combine_kernel     out[t] = sum over slots, in slot order
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "quant_act.cuh"

namespace ql {

// ------------------------------------------------------------------------------ routing
// One warp per token.  logits [T, E] fp32 (E <= 256), k <= 16.
__global__ void __launch_bounds__(256) moe_topk_kernel(const float* __restrict__ logits, int T,
                                                       int E, int k, int* __restrict__ ids,
                                                       float* __restrict__ gates,
                                                       int* __restrict__ counts) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? logits[static_cast<size_t>(warp) * E + e] : -INFINITY;
  }
  float sel[16];
  int sid[16];
  for (int s = 0; s < k; ++s) {
    // lane-local best (largest value, then lowest id)
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E && (v[i] > bv || (v[i] == bv && e < bi))) { bv = v[i]; bi = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
      const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    sel[s] = bv;
    sid[s] = bi;
    if ((bi & 31) == lane) v[bi >> 5] = -INFINITY;   // remove the winner
  }
  if (lane == 0) {
    float sum = 0.f, ex[16];
    for (int s = 0; s < k; ++s) { ex[s] = expf(sel[s] - sel[0]); sum += ex[s]; }
    for (int s = 0; s < k; ++s) {
      ids[static_cast<size_t>(warp) * k + s] = sid[s];
      gates[static_cast<size_t>(warp) * k + s] = ex[s] / sum;
      atomicAdd(&counts[sid[s]], 1);
    }
  }
}

// One CTA (256 threads) per expert e: offsets[e] = sum of counts[<e]; the entries f with
// ids[f] == e are written, ascending, to entries[offsets[e] ...].  CTA 0 also writes offsets[E].
__global__ void __launch_bounds__(256) moe_scatter_kernel(const int* __restrict__ ids, int total,
                                                          int E, const int* __restrict__ counts,
                                                          int* __restrict__ offsets,
                                                          int* __restrict__ entries) {
  const int e = blockIdx.x;
  __shared__ int s_base, s_warp[8];
  if (threadIdx.x == 0) {
    int b = 0;
    for (int i = 0; i < e; ++i) b += counts[i];
    s_base = b;
    offsets[e] = b;
    if (e == 0) offsets[E] = total;
  }
  __syncthreads();
  int pos = s_base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int f0 = 0; f0 < total; f0 += blockDim.x) {
    const int f = f0 + threadIdx.x;
    const bool hit = f < total && ids[f] == e;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, hit);
    if (lane == 0) s_warp[warp] = __popc(m);
    __syncthreads();
    int before = 0, all = 0;
    for (int w = 0; w < 8; ++w) {
      if (w < warp) before += s_warp[w];
      all += s_warp[w];
    }
    if (hit) entries[pos + before + __popc(m & ((1u << lane) - 1u))] = f;
    pos += all;
    __syncthreads();
  }
}

// out[t, n] = sum_{s < k} yslot[(t*k + s), n] in slot order; 4 outputs per thread.
__global__ void __launch_bounds__(256) moe_combine_kernel(const float* __restrict__ yslot, int T,
                                                          int H, int k,
                                                          __nv_bfloat16* __restrict__ out,
                                                          float* __restrict__ out32) {
  const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;   // float4 index
  const long n4 = static_cast<long>(T) * H / 4;
  if (i >= n4) return;
  const long t = (i * 4) / H;
  const int n = static_cast<int>((i * 4) % H);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < k; ++s) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(yslot + (t * k + s) * H + n));
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + t * H + n) = pk;
  if (out32 != nullptr) *reinterpret_cast<float4*>(out32 + t * H + n) = acc;
}

// ------------------------------------------------------------------------------ grouped GEMM
struct MoeGemmArgs {
  int E, k;
  int rows_per_expert;            // weight rows per expert: 2I (gate/up) or H (down)
  int kdim;                       // reduction width: H (gate/up) or I (down)
  int n_tiles;                    // rows_per_expert / 128
  const int* counts;              // [E]
  const int* offsets;             // [E+1]
  const int* entries;             // [T*k] routed entries, expert-sorted
  const __nv_bfloat16* cent;      // [E*rows_per_expert][16] centroids (kernel row order)
  const float* gates;             // [T*k] gate weights by entry (down)
  int I;                          // intermediate width
  uint8_t* h_codes;               // [T*k, I/2] MXFP4 codes of h, sorted order (gate/up)
  uint8_t* h_scales;              // [T*k, I/32] E8M0 bytes
  __nv_bfloat16* h_dq;            // [T*k, I] exact bf16 of the quantized h
  float* h32;                     // optional [T*k, I] fp32 h before quantization
  float* yslot;                   // [T*k, H] gate * y per entry (down)
  int H;
};

template <int BN>
struct MoeCfg {
  static constexpr int kABytes = 128 * 128;       // 128 rows x 64 bf16
  static constexpr int kBBytes = BN * 128;        // BN rows x 64 bf16
  static constexpr int kIdxBytes = 128 * 32;      // 128 rows x 64 4-bit indices
  static constexpr int kStageBytes = kABytes + kBBytes + kIdxBytes;
  static constexpr int kStages = (180 * 1024) / kStageBytes > 6 ? 6 : (180 * 1024) / kStageBytes;
  static constexpr int kCentBytes = 128 * 16 * 2;
  static constexpr int kTmemCols = BN < 32 ? 32 : BN;
  static constexpr int kSmemBytes = kStages * kStageBytes + kCentBytes + BN * 8 + 1024 + 256;
  static_assert(BN * 64 * 4 <= kStages * kStageBytes, "SwiGLU staging must fit the ring");
};

__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3),
      "r"(smem_u32(bar))
      : "memory");
}


// One CTA per work item (expert e, 128-row weight tile nt, BN-token tile mt), items enumerated
// expert by expert, nt fastest.  GATEUP: weight rows of a tile are 64 gate rows then the 64
// matching up rows (repacked at create time), so the SwiGLU pairs meet inside one tile.
template <int BN, bool GATEUP>
__global__ void __launch_bounds__(192, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tm_idx,
                    const __grid_constant__ CUtensorMap tm_b, const MoeGemmArgs a) {
  using Cfg = MoeCfg<BN>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * Cfg::kABytes;
  uint8_t* sIdx = sB + S * Cfg::kBBytes;
  __nv_bfloat16* sCent = reinterpret_cast<__nv_bfloat16*>(sIdx + S * Cfg::kIdxBytes);
  int* sRow = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(sCent) + Cfg::kCentBytes);  // [BN]
  float* sGate = reinterpret_cast<float*>(sRow + BN);                                         // [BN]
  uint64_t* full = reinterpret_cast<uint64_t*>(sGate + BN);
  uint64_t* empty = full + S;
  uint64_t* decd = empty + S;
  uint64_t* cfull = decd + S;
  uint64_t* accf = cfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  int* s_item = reinterpret_cast<int*>(tmem_slot + 1);   // e, nt, mt, count in tile, p0

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    int item = blockIdx.x, base = 0, e = 0;
    for (; e < a.E; ++e) {
      const int it = a.n_tiles * ((a.counts[e] + BN - 1) / BN);
      if (item < base + it) break;
      base += it;
    }
    s_item[0] = e;
    if (e < a.E) {
      const int local = item - base;
      s_item[1] = local % a.n_tiles;
      s_item[2] = local / a.n_tiles;
      s_item[3] = min(BN, a.counts[e] - s_item[2] * BN);
      s_item[4] = a.offsets[e] + s_item[2] * BN;
    }
  }
  __syncthreads();
  const int e = s_item[0];
  if (e >= a.E) return;                                  // past the last item: whole CTA leaves
  const int nt = s_item[1], cnt = s_item[3], p0 = s_item[4];
  const int row0 = e * a.rows_per_expert + nt * 128;
  for (int j = threadIdx.x; j < BN; j += blockDim.x) {
    const int f = j < cnt ? a.entries[p0 + j] : a.entries[p0];
    sRow[j] = GATEUP ? f / a.k : f;
    sGate[j] = GATEUP ? 0.f : a.gates[f];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&decd[s], 128);
    }
    mbar_init(cfull, 1);
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nstages = a.kdim / 64;

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(cfull, Cfg::kCentBytes);
      bulk_load(sCent, a.cent + static_cast<size_t>(row0) * 16, Cfg::kCentBytes, cfull);
      for (int i = 0, it = 0; i < nstages && ok; ++i, ++it) {
        const int st = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!mbar_wait(&empty[st], ph ^ 1, 11)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[st], Cfg::kIdxBytes + Cfg::kBBytes);
        tma_load_2d(sIdx + st * Cfg::kIdxBytes, &tm_idx, &full[st], i * 32, row0);
        if constexpr (GATEUP) {
#pragma unroll 4
          for (int g = 0; g < BN / 4; ++g)
            tma_gather4(sB + st * Cfg::kBBytes + g * 512, &tm_b, &full[st], i * 64, sRow[4 * g],
                        sRow[4 * g + 1], sRow[4 * g + 2], sRow[4 * g + 3]);
        } else {
          tma_load_2d(sB + st * Cfg::kBBytes, &tm_b, &full[st], i * 64, p0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BN);
      for (int i = 0, it = 0; i < nstages && ok; ++i, ++it) {
        const int st = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!mbar_wait(&full[st], ph, 12) || !mbar_wait(&decd[st], ph, 13)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + st * Cfg::kABytes);
        const uint32_t b_base = smem_u32(sB + st * Cfg::kBBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem, make_sdesc(a_base + kk * 32, 16, 1024, kLayoutSW128),
                  make_sdesc(b_base + kk * 32, 16, 1024, kLayoutSW128), idesc,
                  (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[st]);
      }
      tc_commit(accf);
    }
  } else {
    // ---------------- decode: 4-bit indices -> bf16 operand tile through the row centroids
    const int t = threadIdx.x - 64;
    if (!mbar_wait(cfull, 0, 14)) ok = false;
    for (int i = 0, it = 0; i < nstages && ok; ++i, ++it) {
      const int st = it % S;
      const uint32_t ph = (it / S) & 1;
      if (!mbar_wait(&full[st], ph, 15)) { ok = false; break; }
      const uint8_t* idx_s = sIdx + st * Cfg::kIdxBytes;
      uint8_t* a_s = sA + st * Cfg::kABytes;
#pragma unroll 2
      for (int j = 0; j < 8; ++j) {
        const int c = t + 128 * j;
        const int r = c >> 3, kc = c & 7;
        const uint32_t iv = *reinterpret_cast<const uint32_t*>(idx_s + r * 32 + kc * 4);
        const uint16_t* L = reinterpret_cast<const uint16_t*>(sCent) + r * 16;
        uint4 o;
        o.x = L[iv & 15u] | (static_cast<uint32_t>(L[(iv >> 4) & 15u]) << 16);
        o.y = L[(iv >> 8) & 15u] | (static_cast<uint32_t>(L[(iv >> 12) & 15u]) << 16);
        o.z = L[(iv >> 16) & 15u] | (static_cast<uint32_t>(L[(iv >> 20) & 15u]) << 16);
        o.w = L[(iv >> 24) & 15u] | (static_cast<uint32_t>(L[iv >> 28]) << 16);
        *reinterpret_cast<uint4*>(a_s + r * 128 + ((kc ^ (r & 7)) << 4)) = o;
      }
      fence_proxy_async_smem();
      mbar_arrive(&decd[st]);
    }
    // ---------------- epilogue
    const int q = warp & 3;
    if (ok) ok = mbar_wait(accf, 0, 16);
    tc_fence_after();
    if constexpr (GATEUP) {
      float* ubuf = reinterpret_cast<float*>(smem);            // [BN][64] up values
      if (q >= 2 && ok) {
        for (int c = 0; c < BN; c += 8) {
          uint32_t r[8];
          tmem_ld8(tmem + (static_cast<uint32_t>(q * 32) << 16) + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) ubuf[(c + j) * 64 + (q - 2) * 32 + lane] = __uint_as_float(r[j]);
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (q < 2 && ok) {
        const int jf = nt * 64 + q * 32 + lane;                 // intermediate feature
        for (int c = 0; c < BN; c += 8) {
          uint32_t r[8];
          tmem_ld8(tmem + (static_cast<uint32_t>(q * 32) << 16) + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (c + j >= cnt) break;
            const float g = __uint_as_float(r[j]);
            const float u = ubuf[(c + j) * 64 + q * 32 + lane];
            const float h = g / (1.0f + expf(-g)) * u;
            const size_t p = static_cast<size_t>(p0 + c + j);
            if (a.h32 != nullptr) a.h32[p * a.I + jf] = h;
            // MXFP4 requantization of h over this warp's 32 features
            uint32_t am = __float_as_uint(h) & 0x7FFFFFFFu;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
            const int E8 = static_cast<int>(am >> 23);
            const int ex = (E8 == 0) ? -127 : max(E8 - 129, -127);
            const float inv = __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
            const float hn = __shfl_xor_sync(0xFFFFFFFFu, h, 1);
            uint32_t byte = e2m1x2(h * inv, hn * inv);                  // even lane: (h, next)
            byte |= ((__float_as_uint(h) >> 28) & 8u) | ((__float_as_uint(hn) >> 24) & 0x80u);
            const uint32_t nb = __shfl_xor_sync(0xFFFFFFFFu, byte, 1);
            const uint32_t mycode = (lane & 1) ? ((nb >> 4) & 15u) : (byte & 15u);
            if ((lane & 1) == 0) a.h_codes[p * (a.I / 2) + (jf >> 1)] = static_cast<uint8_t>(byte);
            if (lane == 0) a.h_scales[p * (a.I / 32) + (jf >> 5)] = static_cast<uint8_t>(ex + 127);
            // exact value of the quantized element (power-of-two scaling; 2^-127 is subnormal)
            a.h_dq[p * a.I + jf] = __float2bfloat16_rn(ldexpf(e2m1_code_value(mycode), ex));
          }
        }
      }
    } else {
      if (ok) {
        const int n = nt * 128 + q * 32 + lane;                 // output feature of the expert
        for (int c = 0; c < BN; c += 8) {
          uint32_t r[8];
          tmem_ld8(tmem + (static_cast<uint32_t>(q * 32) << 16) + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (c + j >= cnt) break;
            a.yslot[static_cast<size_t>(sRow[c + j]) * a.H + n] = __uint_as_float(r[j]) * sGate[c + j];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace ql
