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
//   moe_gather_kernel      the bf16 row of x for every routed entry, in expert-sorted order
//   moe_gemm_kernel<GATEUP> gate/up: B = the expert's contiguous gathered rows; epilogue
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
  __shared__ int s_hist[256];   // this CTA's routed count per expert (one global add per expert)
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp < T) {
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
      atomicAdd(&s_hist[sid[s]], 1);
    }
  }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (s_hist[e] != 0) atomicAdd(&counts[e], s_hist[e]);
}

// One CTA (1024 threads) per expert e: offsets[e] = sum of counts[<e]; the entries f with
// ids[f] == e are written, ascending, to entries[offsets[e] ...].  CTA 0 also writes offsets[E].
// Each thread tests 16 consecutive entries per pass (a bit mask), a block-wide exclusive scan of
// the hit counts gives every hit its place.
constexpr int kScatterThreads = 1024;
__global__ void __launch_bounds__(kScatterThreads) moe_scatter_kernel(
    const int* __restrict__ ids, int total, int E, const int* __restrict__ counts,
    int* __restrict__ offsets, int* __restrict__ entries) {
  const int e = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_base, s_pass, s_warp[32];
  if (warp == 0) {
    int b = 0;
    for (int i = lane; i < e; i += 32) b += counts[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
    if (lane == 0) {
      s_base = b;
      offsets[e] = b;
      if (e == 0) offsets[E] = total;
    }
  }
  __syncthreads();
  int pos = s_base;
  for (int c0 = 0; c0 < total; c0 += kScatterThreads * 16) {
    const int f0 = c0 + threadIdx.x * 16;
    uint32_t mask = 0;
    if (f0 + 16 <= total && (total & 3) == 0) {
      const int4* src = reinterpret_cast<const int4*>(ids + f0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int4 v = __ldg(src + q);
        mask |= (v.x == e ? 1u : 0u) << (4 * q) | (v.y == e ? 1u : 0u) << (4 * q + 1) |
                (v.z == e ? 1u : 0u) << (4 * q + 2) | (v.w == e ? 1u : 0u) << (4 * q + 3);
      }
    } else {
      for (int j = 0; j < 16; ++j)
        if (f0 + j < total && __ldg(ids + f0 + j) == e) mask |= 1u << j;
    }
    const int cnt = __popc(mask);
    int incl = cnt;   // inclusive scan over the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = s_warp[lane], wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xFFFFFFFFu, wi, o);
        if (lane >= o) wi += u;
      }
      s_warp[lane] = wi - w;   // exclusive prefix of the warps
      if (lane == 31) s_pass = wi;   // hits of this pass
    }
    __syncthreads();
    int at = pos + s_warp[warp] + incl - cnt;
    while (mask != 0) {
      const int j = __ffs(mask) - 1;
      entries[at++] = f0 + j;
      mask &= mask - 1;
    }
    pos += s_pass;
    __syncthreads();   // s_warp and s_pass are rewritten by the next pass
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

// xs[p, :] = x_dq[entries[p] / k, :] for every routed entry p (expert-sorted order), so that each
// expert's activation rows are contiguous and the gate/up GEMM reads them as plain TMA tiles.
// One thread per 16 bytes.
__global__ void __launch_bounds__(256) moe_gather_kernel(const __nv_bfloat16* __restrict__ x_dq,
                                                         const int* __restrict__ entries, int P,
                                                         int H, int k,
                                                         __nv_bfloat16* __restrict__ xs) {
  const long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per_row = H / 8;
  if (i >= static_cast<long>(P) * per_row) return;
  const int p = static_cast<int>(i / per_row), c = static_cast<int>(i - static_cast<long>(p) * per_row);
  const int t = __ldg(entries + p) / k;
  reinterpret_cast<uint4*>(xs + static_cast<size_t>(p) * H)[c] =
      __ldg(reinterpret_cast<const uint4*>(x_dq + static_cast<size_t>(t) * H) + c);
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
  int had;                        // gate/up: online Hadamard (block 32) of h before requantizing
  int H;
};

template <int BN>
struct MoeCfg {
  static constexpr int kABytes = 128 * 128;       // 128 rows x 64 bf16
  static constexpr int kBBytes = BN * 128;        // BN rows x 64 bf16
  static constexpr int kIdxBytes = 128 * 32;      // 128 rows x 64 4-bit indices
  static constexpr int kStageBytes = kABytes + kBBytes + kIdxBytes;
  static constexpr int kStages = BN > 128 ? 3 : 5;
  static constexpr int kCentBytes = 128 * 16 * 2;
  static constexpr int kHalf = 64;                // tokens per epilogue pass
  static constexpr int kStgLd = 129;              // padded row of the transposed staging tile
  static constexpr int kStgBytes = kHalf * kStgLd * 4;
  static constexpr int kTmemCols = 2 * BN;        // two accumulators (ping-pong across items)
  static constexpr int kDecGroups = 3;            // decoder groups, each on every third stage
  static constexpr int kDecWarps = 4 * kDecGroups;
  static constexpr int kThreads = (2 + kDecWarps + 4) * 32;
  static constexpr int kSmemBytes =
      kStages * kStageBytes + 2 * kCentBytes + kStgBytes + 1024 + 512;
  static_assert(kSmemBytes + 5200 <= 227 * 1024, "dynamic + static shared memory per block");
};

// Persistent grouped GEMM.  Work items (expert e, 128-row weight tile nt, BN-token tile mt) are
// enumerated expert by expert, nt fastest; CTA c takes items c, c + gridDim.x, ...  Warp roles:
// 0 producer (TMA: index tile, B rows -- the expert's contiguous gathered x rows for gate/up, its
// h rows for down -- and the item's 128 centroid rows), 1 TMEM allocator + MMA issuer (kind::f16, N = the
// item's token count rounded up to 16), 2 .. 1 + kDecWarps decode (4-bit indices -> bf16 operand
// tile; groups of four warps take the stages round-robin), the last four warps the epilogue.  Two TMEM accumulators alternate between items, so the epilogue of one item
// overlaps the main loop of the next.  GATEUP: the weight rows of a tile are 64 gate rows then
// the 64 matching up rows (repacked at create time), so the SwiGLU pairs meet inside one tile.
template <int BN, bool GATEUP>
__global__ void __launch_bounds__(MoeCfg<BN>::kThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tm_idx,
                    const __grid_constant__ CUtensorMap tm_b, const MoeGemmArgs a) {
  using Cfg = MoeCfg<BN>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  // 1 KB aligned by offsetting the shared array itself, so that every pointer derived from it
  // stays a shared-space pointer (plain ld/st.shared, not generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * Cfg::kABytes;
  uint8_t* sIdx = sB + S * Cfg::kBBytes;
  __nv_bfloat16* sCent = reinterpret_cast<__nv_bfloat16*>(sIdx + S * Cfg::kIdxBytes);    // [2][128][16]
  float* sStg = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sCent) + 2 * Cfg::kCentBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sStg) + Cfg::kStgBytes);   // B rows landed
  uint64_t* ifull = full + S;                                       // index tile landed
  uint64_t* empty = ifull + S;
  uint64_t* decd = empty + S;
  uint64_t* cfull = decd + S;     // [2] centroids + row list of an item landed
  uint64_t* cempty = cfull + 2;   // [2] decoders done with them
  uint64_t* accf = cempty + 2;    // [2] accumulator complete
  uint64_t* acce = accf + 2;      // [2] accumulator drained by the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
  __shared__ int s_pre[257];      // first item of each expert; s_pre[E] = number of items
  __shared__ int s_cnt[256], s_off[256];   // routed token count and first entry of each expert
  __shared__ int s_f[BN];         // down epilogue: routed entry of each token of the item
  __shared__ float s_g[BN];       //                and its gate weight

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    const int c = a.counts[e];
    s_cnt[e] = c;
    s_off[e] = a.offsets[e];
    s_pre[e + 1] = a.n_tiles * ((c + BN - 1) / BN);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ifull[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&decd[s], 4);   // one decoder group (4 warps) per stage
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&cfull[b], 1);
      mbar_init(&cempty[b], Cfg::kDecWarps * 32);
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 128);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    s_pre[0] = 0;
    for (int e = 0; e < a.E; ++e) s_pre[e + 1] += s_pre[e];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = s_pre[a.E];
  const int nstages = a.kdim / 64;

  struct Item { int e, nt, cnt, p0; };
  auto item_of = [&](int id) {
    int lo = 0, hi = a.E - 1;                 // last expert with s_pre[e] <= id
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= id) lo = mid; else hi = mid - 1;
    }
    Item it;
    it.e = lo;
    const int local = id - s_pre[lo];
    it.nt = local % a.n_tiles;
    const int mt = local / a.n_tiles;
    it.cnt = min(BN, s_cnt[lo] - mt * BN);
    it.p0 = s_off[lo] + mt * BN;
    return it;
  };

  bool ok = true;
  if (warp == 0) {
    // ---------------- producer
    int it = 0;   // global stage counter
    for (int id = blockIdx.x, j = 0; id < n_items && ok; id += gridDim.x, ++j) {
      const Item I = item_of(id);
      const int b = j & 1;
      const int row0 = I.e * a.rows_per_expert + I.nt * 128;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&cempty[b], ((j >> 1) & 1) ^ 1, 11));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&cfull[b], Cfg::kCentBytes);
        bulk_load(sCent + b * 128 * 16, a.cent + static_cast<size_t>(row0) * 16, Cfg::kCentBytes, &cfull[b]);
      }
      for (int i = 0; i < nstages && ok; ++i, ++it) {
        const int st = it % S;
        const uint32_t ph = (it / S) & 1;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&empty[st], ph ^ 1, 12));
        if (!ok) break;
        if (lane < 2) {   // both copies in one instruction stream: lane 0 the indices, lane 1 B
          uint64_t* bar = lane == 0 ? &ifull[st] : &full[st];
          mbar_arrive_expect_tx(bar, lane == 0 ? Cfg::kIdxBytes : Cfg::kBBytes);
          tma_load_2d(lane == 0 ? static_cast<void*>(sIdx + st * Cfg::kIdxBytes) : static_cast<void*>(sB + st * Cfg::kBBytes),
                      lane == 0 ? &tm_idx : &tm_b, bar, lane == 0 ? i * 32 : i * 64, lane == 0 ? row0 : I.p0);
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    int it = 0;
    for (int id = blockIdx.x, j = 0; id < n_items && ok; id += gridDim.x, ++j) {
      const Item I = item_of(id);
      const int b = j & 1;
      const int nrow = min(BN, (I.cnt + 15) & ~15);
      const uint32_t idesc = idesc_bf16(nrow);
      const uint32_t acc = tmem + b * BN;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&acce[b], ((j >> 1) & 1) ^ 1, 17));
      if (!ok) break;
      tc_fence_after();
      for (int i = 0; i < nstages && ok; ++i, ++it) {
        const int st = it % S;
        const uint32_t ph = (it / S) & 1;
        // decd: the stage's A tile is decoded and (each decoder warp waited for it) its B tile landed
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&decd[st], ph, 14));
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + st * Cfg::kABytes);
        const uint32_t b_base = smem_u32(sB + st * Cfg::kBBytes);
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(acc, make_sdesc(a_base + kk * 32, 16, 1024, kLayoutSW128),
                    make_sdesc(b_base + kk * 32, 16, 1024, kLayoutSW128), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[st]);
          if (i == nstages - 1) tc_commit(&accf[b]);
        }
        __syncwarp();
      }
    }
  } else if (warp < 2 + Cfg::kDecWarps) {
    // ---------------- decode: 4-bit indices -> bf16 operand tile through the row centroids.
    // kDecGroups groups of four decoder warps take the stages round-robin: a stage's barrier
    // waits, index loads and table lookups cost a group more than the MMAs need, so the groups
    // overlap one another's.
    constexpr int kDT = 128;                                  // threads per group
    const int grp = (warp - 2) / 4;
    const int t = threadIdx.x - 64 - grp * kDT;
    int it = 0;
    for (int id = blockIdx.x, j = 0; id < n_items && ok; id += gridDim.x, ++j) {
      const int b = j & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&cfull[b], (j >> 1) & 1, 15))) { ok = false; break; }
      const uint16_t* cent = reinterpret_cast<const uint16_t*>(sCent + b * 128 * 16);
      for (int i = 0; i < nstages && ok; ++i, ++it) {
        if (it % Cfg::kDecGroups != grp) continue;
        const int st = it % S;
        const uint32_t ph = (it / S) & 1;
        // indices only: runs ahead of B (warp-uniform: the warp leaves the loop together)
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&ifull[st], ph, 16))) { ok = false; break; }
        const uint8_t* idx_s = sIdx + st * Cfg::kIdxBytes;
        uint8_t* a_s = sA + st * Cfg::kABytes;
#pragma unroll
        for (int jj = 0; jj < 1024 / kDT; ++jj) {
          const int c = t + kDT * jj;
          const int r = c >> 3, kc = c & 7;
          const uint32_t iv = *reinterpret_cast<const uint32_t*>(idx_s + r * 32 + kc * 4);
          const uint16_t* L = cent + r * 16;
          uint4 o;
          o.x = L[iv & 15u] | (static_cast<uint32_t>(L[(iv >> 4) & 15u]) << 16);
          o.y = L[(iv >> 8) & 15u] | (static_cast<uint32_t>(L[(iv >> 12) & 15u]) << 16);
          o.z = L[(iv >> 16) & 15u] | (static_cast<uint32_t>(L[(iv >> 20) & 15u]) << 16);
          o.w = L[(iv >> 24) & 15u] | (static_cast<uint32_t>(L[iv >> 28]) << 16);
          *reinterpret_cast<uint4*>(a_s + r * 128 + ((kc ^ (r & 7)) << 4)) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (!mbar_wait(&full[st], ph, 13)) ok = false;
          mbar_arrive(&decd[st]);
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      }
      if (ok) mbar_arrive(&cempty[b]);
    }
  } else {
    // ---------------- epilogue (4 warps; TMEM lane quadrant = warp % 4)
    const int q = warp & 3;
    const int et = threadIdx.x - (2 + Cfg::kDecWarps) * 32;   // 0..127
    const int row = q * 32 + lane;                             // accumulator row of this thread
    for (int id = blockIdx.x, j = 0; id < n_items && ok; id += gridDim.x, ++j) {
      const Item I = item_of(id);
      const int b = j & 1;
      ok = bar_and(2, 128, mbar_wait(&accf[b], (j >> 1) & 1, 18));   // all 128 agree
      if (!ok) break;
      tc_fence_after();
      const uint32_t acc = tmem + b * BN + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (GATEUP) {
        // Transpose half a tile at a time through shared memory ([token][row], padded), then
        // thread et handles token et % kHalf and MX block et / kHalf (32 intermediate features):
        // h = silu(g) * u, MXFP4 requantization, the exact bf16 of the quantized h.
        constexpr int H2 = Cfg::kHalf;
        for (int h0 = 0; h0 < BN; h0 += H2) {
          if (h0 < I.cnt) {
#pragma unroll 1
            for (int c = 0; c < H2; c += 8) {
              uint32_t r[8];
              tmem_ld8(acc + h0 + c, r);
              tmem_ld_wait();
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) sStg[(c + jj) * Cfg::kStgLd + row] = __uint_as_float(r[jj]);
            }
          }
          if (h0 + H2 >= BN) {   // last read of this accumulator
            tc_fence_before();
            mbar_arrive(&acce[b]);
          }
          asm volatile("bar.sync 2, 128;" ::: "memory");
          const int c = et % H2, blk = et / H2;
          if (h0 + c < I.cnt && blk < 2) {
            const float* gr = sStg + c * Cfg::kStgLd + 32 * blk;
            const float* ur = gr + 64;
            float hv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float g = gr[i];
              hv[i] = g / (1.0f + expf(-g)) * ur[i];
            }
            if (a.h32 != nullptr) {   // h as computed, before any rotation (stage-wise checks)
              const size_t p = static_cast<size_t>(I.p0 + h0 + c);
              float4* d32 = reinterpret_cast<float4*>(a.h32 + p * a.I + I.nt * 64 + 32 * blk);
#pragma unroll
              for (int i = 0; i < 8; ++i) d32[i] = make_float4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
            }
            if (a.had) fwht32(hv);   // online Hadamard of h before its requantization
            uint4 c4;
            uint32_t byte;
            code_mx_f32(hv, c4, byte);
            const uint32_t code[4] = {c4.x, c4.y, c4.z, c4.w};
            const int ex = static_cast<int>(byte) - 127;
            const size_t p = static_cast<size_t>(I.p0 + h0 + c);
            const int jf0 = I.nt * 64 + 32 * blk;                  // first intermediate feature
            *reinterpret_cast<uint4*>(a.h_codes + p * (a.I / 2) + jf0 / 2) =
                make_uint4(code[0], code[1], code[2], code[3]);
            a.h_scales[p * (a.I / 32) + jf0 / 32] = static_cast<uint8_t>(ex + 127);
            uint32_t dq[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t c0 = (code[i >> 2] >> (8 * (i & 3))) & 15u;
              const uint32_t c1 = (code[i >> 2] >> (8 * (i & 3) + 4)) & 15u;
              const __nv_bfloat162 v = __floats2bfloat162_rn(ldexpf(e2m1_code_value(c0), ex),
                                                             ldexpf(e2m1_code_value(c1), ex));
              dq[i] = *reinterpret_cast<const uint32_t*>(&v);
            }
            uint4* dst = reinterpret_cast<uint4*>(a.h_dq + p * a.I + jf0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(dq[4 * i], dq[4 * i + 1], dq[4 * i + 2], dq[4 * i + 3]);
          }
          asm volatile("bar.sync 2, 128;" ::: "memory");
        }
      } else {
        // down: y_e[token, n] * gate, scattered to the token's slot row (coalesced along n).
        // The item's routed entries and gates are fetched once, in parallel, into shared memory.
        for (int c = et; c < I.cnt; c += 128) {
          const int f = a.entries[I.p0 + c];
          s_f[c] = f;
          s_g[c] = a.gates[f];
        }
        named_bar_sync(2, 128);
        const int n = I.nt * 128 + row;
#pragma unroll 1
        for (int c = 0; c < I.cnt; c += 8) {
          uint32_t r[8];
          tmem_ld8(acc + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            if (c + jj < I.cnt)
              a.yslot[static_cast<size_t>(s_f[c + jj]) * a.H + n] = __uint_as_float(r[jj]) * s_g[c + jj];
          }
        }
        tc_fence_before();
        mbar_arrive(&acce[b]);
        named_bar_sync(2, 128);   // s_f / s_g are rewritten by the next item
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace ql
