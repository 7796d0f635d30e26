// Decode-size W4A4 GEMM (M <= 64 tokens) on tcgen05, with the activation quantizer fused in.
//
//   y[m, n] = alpha * sum_k x_q[m, k] * w_q[n, k]
//
// The weight forms are those of fp4_gemm_kernel: block-scaled E2M1 with E8M0-B32 scales
// (kind::mxf4, PRQuant tail stages included), with E4M3-B16 scales (kind::mxf4nvf4, alpha = the
// two FP32 tensor scales), or MXCode PreScale VQ indices decoded in shared memory (MXCode
// abstract: MX-native operands rebuilt without a high-precision weight).  At decode sizes the
// layer is bound by streaming the weight, so every CTA owns one 128-row weight tile and a range
// of K stages (split-K), issues the bulk copies of ALL its weight stages at once, keeps them
// resident, and the tokens are one B tile of BN = 16, 32 or 64 rows.
//
// Activation quantization inside the kernel (fuse = 1).  The bf16 activations of split z's
// columns are shared out, in units of 32 elements, among the CTAs of split z; each CTA's four
// quantizer warps quantize their units once (E8M0-B32 per the OCP MX rule PRQuant quantizes
// with, or E4M3-B16 per MXCode Table 1) into the workspace, already in the layout of the MMA's B
// tile of each K stage (128 B per row, 128-byte swizzle) with the stage's scale atoms beside it,
// so that every CTA brings in the B operand of all its stages with two bulk copies.  The E4M3-B16
// tensor scale needs the amax of the whole tensor: each CTA publishes the amax of its units in a
// slot, CTA 0 gathers the slots and publishes the maximum in one word, which the others poll.
// With fuse = 0 the workspace already holds the quantized activations in the plain layout
// (qlinear_quantize_input) and the producer warp copies each stage's B tile with one TMA tile.
//
// Issuing tcgen05 instructions costs the issuing thread tens of cycles each, so the MMA issuer
// issues MMAs only: the scale factors reach TMEM through tcgen05.st from the warps that hold them
// (the decoder, or epilogue, warps for the weight's; the quantizer warps for the activations').
//
// Grid-wide agreement without clearing anything between launches.  The workspace sync block holds
// a launch counter c.  Every CTA reads c once, after griddepcontrol.wait (so after the previous
// launch on the workspace has completed), and tags every word it publishes with tag(c + 1): its
// slot (E4M3: tag | amax), its "units quantized" flag, its "split-K partial written" flag, and
// CTA 0's amax result.  Waiters compare the tag, so stale words of earlier launches never match.
// CTA 0 advances the counter by one at its very end, once it has seen every CTA's slot (so every
// CTA has read c).  A CTA whose bounded wait expired adds two at its end instead: a CTA that read
// the counter late (value v, after CTA 0 gave up) leaves words tagged tag(v + 1) and then the
// counter at v + 2 or more, so the next launch's tag matches no word any failed launch left
// behind, and the workspace stays usable without clearing.
//
// Split-K reduction.  Each CTA of a tile writes its fp32 partial [M][128] to the workspace and
// publishes its flag; every CTA of the tile waits for the tile's flags and reduces 1/S of the
// tile's outputs, adding the splits' partials in split order (deterministic), and writes y.
//
// Warp roles: 0 producer (weight bulk copies, then the B tiles; then the MMA issuer of the odd
// stages into a second accumulator), 1 TMEM allocator + MMA issuer of the even stages,
// VQ: 2..9 decoders (the operand tile of each stage rebuilt from the codebooks into a ring of up
// to eight shared-memory tiles, as many as the memory left by the resident stages holds; warps
// 2..5 also move the stage's weight scales to TMEM), 2..5 epilogue (without VQ they move the
// weight scales), then four quantizer warps.  Every wait is bounded and records the device error
// word.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ptx.cuh"
#include "quant_act.cuh"

namespace ql {

constexpr int kDecMaxGrid = 256;           // CTAs of one decode launch (slots and flags)
constexpr int kDecQUnits = 2;              // 32-element activation units per quantizer thread
constexpr int kDecMaxSplits = 16;          // K-splits of one weight tile
constexpr int kDecLocalBatch = 4;          // local quantization: units a thread loads at once
constexpr int kDecSyncBytes = 16 + 3 * 8 * kDecMaxGrid;

// Workspace sync block: [0] launch counter, [8] amax result, [16..) slots, qflags, pflags (64-bit
// words each).
struct DecSync {
  uint32_t* counter;
  unsigned long long* result;   // CTA 0's published E4M3 amax (tagged)
  unsigned long long* slots;
  unsigned long long* qflags;
  unsigned long long* pflags;
};
__host__ __device__ inline DecSync dec_sync(uint8_t* base) {
  DecSync s;
  s.counter = reinterpret_cast<uint32_t*>(base);
  s.result = reinterpret_cast<unsigned long long*>(base + 8);
  s.slots = reinterpret_cast<unsigned long long*>(base + 16);
  s.qflags = s.slots + kDecMaxGrid;
  s.pflags = s.qflags + kDecMaxGrid;
  return s;
}

// 48-bit tag of a launch count (the low 16 bits of a published word carry data).
__device__ __forceinline__ unsigned long long dec_tag(uint32_t c) {
  return (static_cast<unsigned long long>(c) << 32) |
         (static_cast<unsigned long long>((c * 0x6D2Bu + 0x1F35u) & 0xFFFFu) << 16);
}

// Bounded wait until *p carries `tag` in its upper 48 bits; returns the word (0 on a timeout,
// which also sets the device error word).
__device__ __forceinline__ unsigned long long dec_wait_tag(const unsigned long long* p,
                                                           unsigned long long tag, int site,
                                                           bool& ok) {
  unsigned long long s = ld_acquire_gpu_u64(p);
  if ((s & ~0xFFFFull) == tag) return s;
  const uint64_t t0 = globaltimer_ns(), limit = wait_limit_ns();
  while (true) {
    __nanosleep(32);
    s = ld_acquire_gpu_u64(p);
    if ((s & ~0xFFFFull) == tag) return s;
    if (globaltimer_ns() - t0 > limit) {
      record_error(DEV_TIMEOUT, site);
      ok = false;
      return 0;
    }
  }
}

struct DecodeArgs {
  int M, N;                   // tokens (<= BN), output features
  int C, k_tail;              // activation width; PRQuant tail width (weight width C + k_tail)
  int n_base_stages;          // ceil(C / 256)
  int n_stages_total;         // + ceil(k_tail / 256)
  int spp;                    // K stages per split
  int splits;                 // CTAs per weight tile (consecutive blockIdx)
  int fuse;                   // 0: x quantized by qlinear_quantize_input (plain layout); 1: inside
                              // the kernel, cooperatively (per-stage tiles in the workspace);
                              // 2: inside the kernel, each CTA its own stages (small x)
  const __nv_bfloat16* x;     // fuse: bf16 activations [M, C]
  uint8_t* xq;                // fuse = 0: quantized activation codes [M, C/2] (workspace; read
                              // through the kernel's tensor map, box 128 B x BN rows)
  uint8_t* sfb;               // fuse = 0: activation scale atoms, 128-row group 0, [C / atomK]
  uint8_t* xt;                // fuse = 1: per K stage the B tile [BN][128 B], 128-byte swizzle
  uint8_t* st;                // fuse = 1: per K stage its activation scale atoms
  float* ts_x;                // E4M3: activation tensor scale (fuse: written; else read)
  float alpha;                // host factor (weight tensor scale, or 1)
  const uint8_t* wt;          // weight blocks [N/128][n_stages_total][kWBytes]
  __nv_bfloat16* y;           // [M, ldy]
  float* y32;                 // optional [M, ldy]
  int ldy;
  float* partials;            // splits > 1: [grid][BN][128] fp32 (rows < M written)
  uint8_t* sync;              // DecSync block
  const uint8_t* scb;         // VQ PreScale+: scale codebook [256][8] E4M3 bytes
  int had;                    // fuse, E8M0: online Hadamard (block 32) before quantizing x
  int amax_coop;              // fuse = 2, E4M3: the tensor amax combined over the CTAs (each
                              // reads a share of x), else every CTA reads all of x
  int act_aug;                // fuse = 0: the plain layout is augmented ([M, C + k_tail], the
                              // tail copied behind): tail stages read coordinate C + j
  int cluster;                // the K-splits of a weight tile form one thread-block cluster: the
                              // split-K partials and the E4M3 amax meet in distributed shared
                              // memory, and the workspace sync block is not used
};

// SF (VQ only): the weight's scales as in Fp4Cfg -- 0 PreScale atoms in the block, 1 PostScale
// (8 QBlock bytes per stage), 2 PreScale+ (2 scale indices per row into a 256 x 8 codebook).
template <int BN, bool E8M0, bool VQ, int SF = 0>
struct DecCfg {
  static constexpr int kDecWarps = VQ ? 8 : 0;
  static constexpr int kQWarp0 = VQ ? 10 : 6;
  static constexpr int kThreads = (kQWarp0 + 4) * 32;
  static constexpr int kAtomK = E8M0 ? 128 : 64;     // K elements per scale atom
  static constexpr int kAtoms = 256 / kAtomK;        // scale atoms per 256-K stage
  static constexpr int kABytes = 128 * 128;          // decoded E2M1 tile, 128 rows x 256 K
  static constexpr int kBBytes = BN * 128;
  static constexpr int kSfBytes = kAtoms * 512;
  static constexpr int kIdxBytes = VQ ? 128 * 64 : 0;
  static constexpr int kLutBytes = VQ ? 8 * 512 : 0;
  static_assert(SF == 0 || (VQ && !E8M0), "PostScale / PreScale+ scales: VQ E4M3-B16 weights");
  static constexpr int kSfTail = SF == 0 ? kSfBytes : SF == 1 ? 16 : 256;
  static constexpr int kWBytes = (VQ ? kIdxBytes + kLutBytes : kABytes) + kSfTail;   // in HBM
  static constexpr int kWStride = (kWBytes + 1023) / 1024 * 1024;                     // in smem
  static constexpr int kScbBytes = SF == 2 ? 2048 : 0;
  static constexpr int kSfaOff = VQ ? kIdxBytes + kLutBytes : kABytes;
  static constexpr int kPerStage = kWStride + kBBytes + kSfBytes;
  static constexpr int kSmemBytes = 226 * 1024;      // dynamic shared memory of the launch
  static constexpr int kData = kSmemBytes - 2048 - kScbBytes;   // minus slack, barriers, codebook
  static constexpr int kMaxRing = 8;                 // VQ: decoded operand tiles in flight
  static constexpr int kSfCols = kAtoms * 4;         // TMEM columns of one scale set
  static constexpr int kMaxStagesTmem = (512 - 2 * BN) / (2 * kSfCols);   // two accumulators
  static constexpr int kMaxStagesSmem = (kData - (VQ ? kABytes : 0)) / kPerStage;
  static constexpr int kMaxStagesRaw = kMaxStagesSmem < kMaxStagesTmem ? kMaxStagesSmem : kMaxStagesTmem;
  static constexpr int kMaxStages = kMaxStagesRaw > 16 ? 16 : kMaxStagesRaw;
  static_assert(kMaxStages >= 2, "decode stages");
  static_assert(kBBytes % 1024 == 0 && kSfBytes % 1024 == 0, "1 KB regions");
  // ring of decoded operand tiles for n_it resident stages: what the shared memory left holds
  __host__ __device__ static constexpr int ring(int n_it) {
    return !VQ ? 0 : ((kData - n_it * kPerStage) / kABytes < kMaxRing
                          ? ((kData - n_it * kPerStage) / kABytes < n_it ? (kData - n_it * kPerStage) / kABytes : n_it)
                          : (kMaxRing < n_it ? kMaxRing : n_it));
  }
};

// MX E8M0-B32 coding of one 32-element unit held as 16 bf16x2 words: codes (16 bytes) and the
// E8M0 byte (OCP MX: e = floor(log2 amax) - 2 from the bf16 exponent, clamped to [-127, 127]).
__device__ __forceinline__ void dec_code_mx(const uint32_t (&w)[16], uint4& codes, uint32_t& byte) {
  uint32_t mx = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) mx = __vmaxu2(mx, w[i] & 0x7FFF7FFFu);
  const uint32_t amax16 = max(mx & 0xFFFFu, mx >> 16);
  const int E = static_cast<int>(amax16 >> 7);
  const int e = (E == 0) ? -127 : max(E - 129, -127);
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);   // 2^-e
  uint32_t packed[4];
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
  codes = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  byte = static_cast<uint32_t>(e + 127);
}

// Four outputs y[m, nn .. nn + 3] = alpha * acc (bf16, and fp32 when requested).
__device__ __forceinline__ void dec_store4(const DecodeArgs& a, int m, int nn, float4 acc, float alpha) {
  const float o4[4] = {acc.x * alpha, acc.y * alpha, acc.z * alpha, acc.w * alpha};
  const size_t o = static_cast<size_t>(m) * a.ldy + nn;
  if (nn + 3 < a.N && (a.ldy & 3) == 0) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(o4[0], o4[1]);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(o4[2], o4[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(a.y + o) = pk;
    if (a.y32 != nullptr) *reinterpret_cast<float4*>(a.y32 + o) = make_float4(o4[0], o4[1], o4[2], o4[3]);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (nn + j < a.N) {
        a.y[o + j] = __float2bfloat16_rn(o4[j]);
        if (a.y32 != nullptr) a.y32[o + j] = o4[j];
      }
  }
}

template <int BN, bool E8M0, bool VQ, int SF = 0>
__global__ void __launch_bounds__(DecCfg<BN, E8M0, VQ, SF>::kThreads, 1)
    fp4_decode_kernel(const __grid_constant__ CUtensorMap tm_x, const DecodeArgs a) {
  using Cfg = DecCfg<BN, E8M0, VQ, SF>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tile = blockIdx.x / a.splits, z = blockIdx.x - tile * a.splits;
  const int T = gridDim.x / a.splits;          // weight tiles
  const int s_begin = z * a.spp;
  const int n_it = max(0, min(a.n_stages_total, s_begin + a.spp) - s_begin);   // <= kMaxStages
  // layout (1 KB regions): weight blocks [n_it], B tiles [n_it], SFB sets [n_it], the ring of
  // decoded operand tiles (VQ); barriers in the last 1 KB
  const int R = Cfg::ring(n_it);
  uint8_t* sW = smem;
  uint8_t* sB = sW + n_it * Cfg::kWStride;
  uint8_t* sSfb = sB + n_it * Cfg::kBBytes;
  uint8_t* sA = sSfb + n_it * Cfg::kSfBytes;
  uint8_t* sScb = smem + Cfg::kData;          // SF 2: the scale codebook
  uint64_t* wfull = reinterpret_cast<uint64_t*>(sScb + Cfg::kScbBytes);
  uint64_t* sfa_ok = wfull + Cfg::kMaxStages;  // weight scales of stage i in TMEM (4 warps)
  uint64_t* decd = sfa_ok + Cfg::kMaxStages;   // VQ: ring slot decoded (8 decoder warps)
  uint64_t* aempty = decd + Cfg::kMaxRing;     // VQ: ring slot consumed by the MMAs
  uint64_t* accf = aempty + Cfg::kMaxRing;
  uint64_t* xready = accf + 1;                 // quantized activations visible (quantizer warps)
  uint64_t* bfull = xready + 1;                // every B tile + SFB set in shared memory
  uint64_t* sfb_ok = bfull + 1;                // activation scales in TMEM (4 quantizer warps)
  uint64_t* scbar = sfb_ok + 1;                // SF 2: the scale codebook landed
  uint64_t* camax = scbar + 1;                 // cluster: every split's amax share arrived
  uint64_t* cpart = camax + 1;                 // cluster: every split's partial is in its smem
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cpart + 1);
  __shared__ uint32_t s_cnt;
  __shared__ uint32_t s_red[4];
  __shared__ float s_ts;
  __shared__ int s_allseen;
  __shared__ int s_fail;   // some bounded wait of this CTA expired
  __shared__ uint32_t s_camax[kDecMaxSplits];   // cluster: the amax share of each split
  griddep_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = tile * 128;
  const DecSync sy = dec_sync(a.sync);
  const uint32_t quad_lanes = static_cast<uint32_t>((warp & 3) * 32) << 16;   // TMEM lane quadrant

  auto stage_coords = [&](int i, int& kw, int& kx, int& valid) {
    if (i < a.n_base_stages) {
      kw = i * 256;
      kx = kw;
      valid = min(256, a.C - kw);
    } else {
      const int j = (i - a.n_base_stages) * 256;
      kw = a.C + j;
      kx = a.C - a.k_tail + j;
      valid = min(256, a.k_tail - j);
    }
  };
  // TMEM columns: accumulators [0, BN) (even stages) and [BN, 2 BN) (odd stages), then per stage
  // the weight's and the activation's scales
  auto sfa_col = [&](int it) { return static_cast<uint32_t>(2 * BN + it * 2 * Cfg::kSfCols); };
  auto sfb_col = [&](int it) { return static_cast<uint32_t>(2 * BN + it * 2 * Cfg::kSfCols + Cfg::kSfCols); };

  if (warp == 0) {
    for (int s = lane; s < Cfg::kMaxStages; s += 32) {
      mbar_init(&wfull[s], 1);
      mbar_init(&sfa_ok[s], 4);
    }
    if (lane < Cfg::kMaxRing) {
      mbar_init(&decd[lane], Cfg::kDecWarps > 0 ? Cfg::kDecWarps : 1);
      mbar_init(&aempty[lane], 1);
    }
    if (lane == 0) {
      mbar_init(accf, 2);   // one commit per MMA issuer
      mbar_init(xready, 1);
      mbar_init(bfull, 1);
      mbar_init(sfb_ok, 4);
      mbar_init(scbar, 1);
      mbar_init(camax, a.splits);
      mbar_init(cpart, a.splits);
      s_fail = 0;
      s_allseen = 0;
    }
    fence_mbar_init();
    __syncwarp();
    if (lane == 0) {   // every weight stage of this CTA at once, before the block-wide barrier
      if constexpr (SF == 2) {
        mbar_arrive_expect_tx(scbar, Cfg::kScbBytes);
        bulk_load(sScb, a.scb, Cfg::kScbBytes, scbar);
      }
      for (int it = 0; it < n_it; ++it) {
        const uint8_t* blk = a.wt + (static_cast<size_t>(tile) * a.n_stages_total + s_begin + it) * Cfg::kWBytes;
        mbar_arrive_expect_tx(&wfull[it], Cfg::kWBytes);
        bulk_load(sW + it * Cfg::kWStride, blk, Cfg::kWBytes, &wfull[it]);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  if (a.cluster) cluster_sync_all();   // every CTA of the cluster has its barriers initialised
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int S = a.splits;

  bool ok = true;
  // ---------------- MMA issuer j (MMAs only: the scale factors are placed by other warps): the
  // stages of parity j into accumulator j.  Warp 1 and, once its copies are issued, warp 0.
  auto mma_issue = [&](int j) {
    const uint32_t idesc0 = idesc_fp4_block(BN, E8M0);
    const uint32_t dacc = tmem + j * BN;
    ok = __all_sync(0xFFFFFFFFu, mbar_wait(sfb_ok, 0, 52)) && ok;
    for (int it = j; it < n_it && ok; it += 2) {
      const int slot = VQ ? it % R : 0;
      // VQ: the decoder warps that place the weight scales arrive on decd only after their
      // tcgen05.st completed, so one wait covers both
      const bool w = VQ ? mbar_wait(&decd[slot], (it / R) & 1, 53) : mbar_wait(&sfa_ok[it], 0, 51);
      ok = __all_sync(0xFFFFFFFFu, w);
      if (!ok) break;
      tc_fence_after();
      int kw, kx, valid;
      stage_coords(s_begin + it, kw, kx, valid);
      const uint32_t ta = tmem + sfa_col(it), tb = tmem + sfb_col(it);
      const uint32_t a_base = VQ ? smem_u32(sA + slot * Cfg::kABytes) : smem_u32(sW + it * Cfg::kWStride);
      const uint32_t b_base = smem_u32(sB + it * Cfg::kBBytes);
      const int nk = valid / 64;
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          if (kk < nk) {
            const int at = (kk * 64) / Cfg::kAtomK;
            const uint32_t byte = E8M0 ? static_cast<uint32_t>((kk & 1) * 2) : 0u;
            const uint64_t ad = make_sdesc(a_base + kk * 32, 16, 1024, kLayoutSW128);
            const uint64_t bd = make_sdesc(b_base + kk * 32, 16, 1024, kLayoutSW128);
            const uint32_t idd = idesc0 | (byte << 29) | (byte << 4);
            const uint32_t sa = (ta + at * 4) | (byte << 30);
            const uint32_t sb = (tb + at * 4) | (byte << 30);
            const uint32_t acc = (it == j && kk == 0) ? 0u : 1u;
            if (E8M0)
              mma_mxf4_block32(dacc, ad, bd, idd, sa, sb, acc);
            else
              mma_nvf4_block16(dacc, ad, bd, idd, sa, sb, acc);
          }
        if (VQ && it + R < n_it) tc_commit(&aempty[slot]);   // the slot may be rewritten once these complete
      }
      __syncwarp();
    }
    if (lane == 0) tc_commit(accf);
    __syncwarp();
  };
  if (warp == 0) {
    // ---------------- the B operand of every stage, once the activations are quantized (the
    // local mode writes it into shared memory directly)
    if (a.fuse != 2) ok = __all_sync(0xFFFFFFFFu, mbar_wait(xready, 0, 50));
    if (a.fuse == 1) {
      // stage tiles and scale sets of this CTA's stages are contiguous in the workspace
      if (lane == 0) {
        const uint32_t bbytes = n_it * Cfg::kBBytes, sbytes = n_it * Cfg::kSfBytes;
        if (ok && n_it > 0) {
          fence_proxy_async_global();   // other CTAs' generic stores, acquired, before async reads
          mbar_arrive_expect_tx(bfull, bbytes + sbytes);
          bulk_load(sB, a.xt + static_cast<size_t>(s_begin) * Cfg::kBBytes, bbytes, bfull);
          bulk_load(sSfb, a.st + static_cast<size_t>(s_begin) * Cfg::kSfBytes, sbytes, bfull);
        } else {
          mbar_arrive(bfull);
        }
      }
    } else if (a.fuse == 0) {
      // plain layout (qlinear_quantize_input): each stage's B tile by one TMA tile (128-byte
      // swizzle; rows past M and columns past C read as zeros), then its scale atoms by one bulk
      // copy, all on one barrier
      if (lane == 0) {
        uint32_t bytes = 0;
        for (int it = 0; it < n_it; ++it) {
          int kw, kx, valid;
          stage_coords(s_begin + it, kw, kx, valid);
          bytes += Cfg::kBBytes + (valid / Cfg::kAtomK) * 512;
        }
        if (ok && n_it > 0) {
          mbar_arrive_expect_tx(bfull, bytes);
          for (int it = 0; it < n_it; ++it) {
            int kw, kx, valid;
            stage_coords(s_begin + it, kw, kx, valid);
            if (a.act_aug) kx = kw;
            tma_load_2d(sB + it * Cfg::kBBytes, &tm_x, bfull, kx >> 1, 0);
            const int nat = valid / Cfg::kAtomK;
            if (nat > 0)
              bulk_load(sSfb + it * Cfg::kSfBytes, a.sfb + static_cast<size_t>(kx / Cfg::kAtomK) * 512,
                        nat * 512, bfull);
          }
        } else {
          mbar_arrive(bfull);
        }
      }
    }
    mma_issue(1);
  } else if (warp == 1) {
    mma_issue(0);
  } else if (warp >= Cfg::kQWarp0) {
    // ---------------- quantizer warps
    const int tq = threadIdx.x - Cfg::kQWarp0 * 32;   // 0..127
    const int G = gridDim.x;
    griddep_wait();   // x, the workspace and the counter follow the grids before this one
    if (tq == 0) s_cnt = a.cluster ? 0u : *reinterpret_cast<volatile uint32_t*>(sy.counter);
    if (a.fuse == 2) {
      // ---- local: this CTA reads all of x for the E4M3 tensor amax (no agreement needed) and
      // quantizes the activations of its own stages straight into their shared-memory B tiles
      // The E4M3 tensor amax: all of x read by every CTA (small x); or, in a cluster, each split
      // reads the x columns of its own stages (together the splits cover x) and the shares meet
      // in distributed shared memory; or, without a cluster, each CTA reads a share of x,
      // publishes it in its slot, and CTA 0 gathers the slots and publishes one word that the
      // others poll.
      const bool xchg = !E8M0 && a.amax_coop && a.cluster;
      const bool gather = !E8M0 && a.amax_coop && !a.cluster;
      float ts = 1.f;
      uint32_t mx = 0;
      if constexpr (!E8M0) {
        if (xchg) {
          const int units = n_it * a.M * 8;
          for (int u0 = tq; u0 < units; u0 += 128 * 4) {
            uint4 v[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int u = u0 + 128 * j;
              int kw, kx, valid, it = 0, m = 0, kc = 0;
              if (u < units) {
                it = u / (a.M * 8);
                const int rem = u - it * (a.M * 8);
                m = rem >> 3;
                kc = rem & 7;
              }
              stage_coords(s_begin + it, kw, kx, valid);
              const bool in = u < units && kc * 32 < valid;
              const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(m) * a.C + kx + kc * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i) v[j][i] = in ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                mx = __vmaxu2(mx, v[j][i].x & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, v[j][i].y & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, v[j][i].z & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, v[j][i].w & 0x7FFF7FFFu);
              }
          }
        } else {
          const long n16 = static_cast<long>(a.M) * a.C / 8;
          const long e0 = gather ? n16 * blockIdx.x / G : 0, e1 = gather ? n16 * (blockIdx.x + 1) / G : n16;
          const uint4* xv = reinterpret_cast<const uint4*>(a.x);
          for (long base = e0 + tq; base < e1; base += 128 * 8) {
            uint4 v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const long i = base + 128L * j;
              v[j] = i < e1 ? __ldg(xv + i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              mx = __vmaxu2(mx, v[j].x & 0x7FFF7FFFu);
              mx = __vmaxu2(mx, v[j].y & 0x7FFF7FFFu);
              mx = __vmaxu2(mx, v[j].z & 0x7FFF7FFFu);
              mx = __vmaxu2(mx, v[j].w & 0x7FFF7FFFu);
            }
          }
        }
      }
      uint32_t m16 = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m16 = max(m16, __shfl_xor_sync(0xFFFFFFFFu, m16, o));
      if (lane == 0) s_red[tq >> 5] = m16;
      named_bar_sync(2, 128);   // s_cnt and s_red
      const uint32_t cnt = s_cnt;
      const unsigned long long tag = dec_tag(cnt + 1u);
      uint32_t amax16 = max(max(s_red[0], s_red[1]), max(s_red[2], s_red[3]));
      if (!a.cluster && tq == 0 && !withheld(blockIdx.x))
        st_release_gpu_u64(&sy.slots[blockIdx.x], tag | (gather ? amax16 : 0u));
      bool qok = true;
      if (gather && blockIdx.x == 0) {
        uint32_t a16 = 0;
        for (int c = tq; c < G; c += 128)
          a16 = max(a16, static_cast<uint32_t>(dec_wait_tag(&sy.slots[c], tag, 54, qok) & 0xFFFFull));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a16 = max(a16, __shfl_xor_sync(0xFFFFFFFFu, a16, o));
        named_bar_sync(2, 128);   // s_red was read above
        if (lane == 0) s_red[tq >> 5] = a16;
        qok = bar_and(2, 128, qok);
        amax16 = max(max(s_red[0], s_red[1]), max(s_red[2], s_red[3]));
        if (tq == 0) {
          s_allseen = qok ? 1 : 0;
          if (qok && !withheld(0)) st_release_gpu_u64(sy.result, tag | amax16);
        }
      } else if (gather) {
        named_bar_sync(2, 128);   // s_red was read above
        if (tq == 0) s_red[0] = static_cast<uint32_t>(dec_wait_tag(sy.result, tag, 61, qok) & 0xFFFFull);
        qok = bar_and(2, 128, qok);
        amax16 = s_red[0];
      } else if (xchg) {
        // this split's share into slot z of every split's s_camax, then an arrival on its barrier
        if (tq < S && !withheld(blockIdx.x)) {
          st_shared_cluster_u32(map_shared_rank(smem_u32(&s_camax[z]), tq), amax16);
          mbar_arrive_remote(map_shared_rank(smem_u32(camax), tq));
        }
        bool w = true;
        if (tq == 0) w = mbar_wait_cluster(camax, 0, 64);
        qok = bar_and(2, 128, w);
        if (qok)
          for (int r = 0; r < S; ++r) amax16 = max(amax16, s_camax[r]);
      }
      if constexpr (!E8M0) ts = tensor_scale_from_amax16(amax16);
      // (stage, row, 32-element chunk) units, kDecLocalBatch per thread loaded at once so that
      // their L2 latencies overlap
      const int units = qok ? n_it * a.M * 8 : 0;
      for (int u0 = tq; u0 < units; u0 += 128 * kDecLocalBatch) {
        uint32_t w[kDecLocalBatch][16];
        int dst[kDecLocalBatch];   // it * 4096 + m * 8 + kc, or -1
#pragma unroll
        for (int j = 0; j < kDecLocalBatch; ++j) {
          const int u = u0 + 128 * j;
          dst[j] = -1;
          if (u < units) {
            const int it = u / (a.M * 8), rem = u - it * (a.M * 8), m = rem >> 3, kc = rem & 7;
            int kw, kx, valid;
            stage_coords(s_begin + it, kw, kx, valid);
            if (kc * 32 < valid) {
              dst[j] = it * 4096 + m * 8 + kc;
              const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(m) * a.C + kx + kc * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint4 v = __ldg(src + i);
                w[j][4 * i] = v.x; w[j][4 * i + 1] = v.y; w[j][4 * i + 2] = v.z; w[j][4 * i + 3] = v.w;
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < kDecLocalBatch; ++j) {
          if (dst[j] < 0) continue;
          const int it = dst[j] >> 12, m = (dst[j] >> 3) & 511, kc = dst[j] & 7;
          uint4 codes;
          uint32_t sbytes;
          if constexpr (E8M0) {
            if (a.had) {
              float v[32];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                v[2 * i] = __uint_as_float(w[j][i] << 16);
                v[2 * i + 1] = __uint_as_float(w[j][i] & 0xFFFF0000u);
              }
              fwht32(v);
              code_mx_f32(v, codes, sbytes);
            } else {
              dec_code_mx(w[j], codes, sbytes);
            }
          } else {
            uint32_t p0[2], p1[2], b0, b1;
            const uint32_t w0[8] = {w[j][0], w[j][1], w[j][2], w[j][3], w[j][4], w[j][5], w[j][6], w[j][7]};
            const uint32_t w1[8] = {w[j][8], w[j][9], w[j][10], w[j][11], w[j][12], w[j][13], w[j][14], w[j][15]};
            quant_e4m3_code_block(w0, ts, p0, b0);
            quant_e4m3_code_block(w1, ts, p1, b1);
            codes = make_uint4(p0[0], p0[1], p1[0], p1[1]);
            sbytes = b0 | (b1 << 8);
          }
          *reinterpret_cast<uint4*>(sB + it * Cfg::kBBytes + m * 128 + ((kc ^ (m & 7)) << 4)) = codes;
          uint8_t* sft = sSfb + it * Cfg::kSfBytes + (m & 31) * 16 + ((m >> 5) & 3) * 4;
          if constexpr (E8M0) {
            sft[(kc >> 2) * 512 + (kc & 3)] = static_cast<uint8_t>(sbytes);
          } else {
            const int j0 = 2 * kc;
            sft[(j0 >> 2) * 512 + (j0 & 3)] = static_cast<uint8_t>(sbytes);
            sft[((j0 + 1) >> 2) * 512 + ((j0 + 1) & 3)] = static_cast<uint8_t>(sbytes >> 8);
          }
        }
      }
      if (!E8M0 && blockIdx.x == 0 && tq == 0 && a.ts_x != nullptr) *a.ts_x = ts;
      fence_proxy_async_smem();   // the B tiles, for the tensor core
      named_bar_sync(2, 128);     // every scale byte is in shared memory
      for (int it = 0; it < n_it; ++it)
        tmem_st_scale_atoms<Cfg::kAtoms>(tmem + quad_lanes + sfb_col(it), sSfb + it * Cfg::kSfBytes, lane);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sfb_ok);
      if (tq == 0) {
        s_ts = ts;
        if (qok) mbar_arrive(xready);   // else the epilogue's bounded wait records the failure
        else s_fail = 1;
      }
      if (!a.cluster && blockIdx.x == 0 && !gather) {   // every slot before CTA 0 advances the counter
        bool sok = true;
        for (int c = tq; c < static_cast<int>(gridDim.x) && sok; c += 128) dec_wait_tag(&sy.slots[c], tag, 54, sok);
        sok = bar_and(2, 128, sok);
        if (tq == 0) {
          s_allseen = sok ? 1 : 0;
          if (!sok) s_fail = 1;
        }
      }
    } else {
    named_bar_sync(2, 128);
    const uint32_t cnt = s_cnt;
    const unsigned long long tag = dec_tag(cnt + 1u);
    // this CTA's units: the columns of split z's base stages, rows shared out over its T tiles
    const int c0 = min(a.C, s_begin * 256);
    const int c1 = min(a.C, min(s_begin + a.spp, a.n_base_stages) * 256);
    const int upr = max(0, c1 - c0) >> 5;                 // 32-element units per row
    const long U = static_cast<long>(a.M) * upr;
    const long u0 = U * tile / T, u1 = U * (tile + 1) / T;
    uint32_t w[kDecQUnits][16];
    uint32_t mx = 0;
    if (a.fuse) {
#pragma unroll
      for (int k = 0; k < kDecQUnits; ++k) {
        const long u = u0 + tq + k * 128;
        if (u < u1) {
          const int m = static_cast<int>(u / upr), j = (c0 >> 5) + static_cast<int>(u - static_cast<long>(m) * upr);
          const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(m) * a.C) + j * 4;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldg(src + i);
            w[k][4 * i] = v.x; w[k][4 * i + 1] = v.y; w[k][4 * i + 2] = v.z; w[k][4 * i + 3] = v.w;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) mx = __vmaxu2(mx, w[k][i] & 0x7FFF7FFFu);
        }
      }
    }
    uint32_t m16 = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m16 = max(m16, __shfl_xor_sync(0xFFFFFFFFu, m16, o));
    if (lane == 0) s_red[tq >> 5] = m16;
    named_bar_sync(2, 128);
    if (!a.cluster && tq == 0 && !withheld(blockIdx.x))   // this CTA has read the counter; E4M3: its amax
      st_release_gpu_u64(&sy.slots[blockIdx.x], tag | max(max(s_red[0], s_red[1]), max(s_red[2], s_red[3])));
    bool qok = true;
    float ts = 1.f;
    // CTA 0 gathers every slot: for the E4M3 tensor amax (then at once), and to know that every
    // CTA has read the counter (without an amax to agree on, at its end)
    const bool amax_needed = a.fuse && !E8M0;
    if (blockIdx.x == 0 && amax_needed) {
      uint32_t a16 = 0;
      for (int c = tq; c < G; c += 128)
        a16 = max(a16, static_cast<uint32_t>(dec_wait_tag(&sy.slots[c], tag, 54, qok) & 0xFFFFull));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a16 = max(a16, __shfl_xor_sync(0xFFFFFFFFu, a16, o));
      named_bar_sync(2, 128);   // s_red was read above
      if (lane == 0) s_red[tq >> 5] = a16;
      qok = bar_and(2, 128, qok);
      const uint32_t amax16 = max(max(s_red[0], s_red[1]), max(s_red[2], s_red[3]));
      if (tq == 0) {
        s_allseen = qok ? 1 : 0;
        if (qok && amax_needed && !withheld(0)) st_release_gpu_u64(sy.result, tag | amax16);
      }
      ts = tensor_scale_from_amax16(amax16);
    } else if (amax_needed) {
      if (tq == 0) s_red[0] = static_cast<uint32_t>(dec_wait_tag(sy.result, tag, 61, qok) & 0xFFFFull);
      qok = bar_and(2, 128, qok);
      ts = tensor_scale_from_amax16(s_red[0]);
    }
    if (a.fuse) {
      if (qok) {
        // codes and scales straight into the stage tiles: unit (m, j) of base stage i = j / 8 goes
        // to chunk j % 8 of row m; PRQuant tail channels also to their tail stage
#pragma unroll
        for (int k = 0; k < kDecQUnits; ++k) {
          const long u = u0 + tq + k * 128;
          if (u < u1) {
            const int m = static_cast<int>(u / upr), j = (c0 >> 5) + static_cast<int>(u - static_cast<long>(m) * upr);
            uint4 codes;
            uint32_t sbytes;   // E8M0: one byte; E4M3: two (blocks 2j, 2j + 1)
            if constexpr (E8M0) {
              if (a.had) {   // online Hadamard of the 32-element block, then its MX coding
                float v[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  v[2 * i] = __uint_as_float(w[k][i] << 16);
                  v[2 * i + 1] = __uint_as_float(w[k][i] & 0xFFFF0000u);
                }
                fwht32(v);
                code_mx_f32(v, codes, sbytes);
              } else {
                dec_code_mx(w[k], codes, sbytes);
              }
            } else {
              uint32_t p0[2], p1[2], b0, b1;
              const uint32_t w0[8] = {w[k][0], w[k][1], w[k][2], w[k][3], w[k][4], w[k][5], w[k][6], w[k][7]};
              const uint32_t w1[8] = {w[k][8], w[k][9], w[k][10], w[k][11], w[k][12], w[k][13], w[k][14], w[k][15]};
              quant_e4m3_code_block(w0, ts, p0, b0);
              quant_e4m3_code_block(w1, ts, p1, b1);
              codes = make_uint4(p0[0], p0[1], p1[0], p1[1]);
              sbytes = b0 | (b1 << 8);
            }
            const int c = j * 32;
            for (int copy = 0; copy < 2; ++copy) {
              int stage, kc;
              if (copy == 0) {
                stage = c >> 8;
                kc = (c & 255) >> 5;
              } else {
                if (a.k_tail == 0 || c < a.C - a.k_tail) break;
                const int t = c - (a.C - a.k_tail);
                stage = a.n_base_stages + (t >> 8);
                kc = (t & 255) >> 5;
              }
              *reinterpret_cast<uint4*>(a.xt + static_cast<size_t>(stage) * Cfg::kBBytes + m * 128 +
                                        ((kc ^ (m & 7)) << 4)) = codes;
              uint8_t* sft = a.st + static_cast<size_t>(stage) * Cfg::kSfBytes + (m & 31) * 16 + ((m >> 5) & 3) * 4;
              if constexpr (E8M0) {
                sft[(kc >> 2) * 512 + (kc & 3)] = static_cast<uint8_t>(sbytes);
              } else {
                const int j0 = 2 * kc;   // 16-element blocks 2kc, 2kc + 1 of the stage
                sft[(j0 >> 2) * 512 + (j0 & 3)] = static_cast<uint8_t>(sbytes);
                sft[((j0 + 1) >> 2) * 512 + ((j0 + 1) & 3)] = static_cast<uint8_t>(sbytes >> 8);
              }
            }
          }
        }
        if (!E8M0 && blockIdx.x == 0 && tq == 0 && a.ts_x != nullptr) *a.ts_x = ts;
      }
      named_bar_sync(2, 128);   // every thread's codes are written before the release below
      if (tq == 0 && qok && !withheld(blockIdx.x)) st_release_gpu_u64(&sy.qflags[blockIdx.x], tag | 1u);
      // the CTAs that quantized this CTA's columns: those of split z, and for PRQuant tail stages
      // every CTA (the tail channels sit in the last base stages)
      const bool tail = s_begin + n_it > a.n_base_stages && a.k_tail > 0;
      if (tail) {
        for (int c = tq; c < G && qok; c += 128) dec_wait_tag(&sy.qflags[c], tag, 55, qok);
      } else {
        for (int t = tq; t < T && qok; t += 128) dec_wait_tag(&sy.qflags[t * a.splits + z], tag, 55, qok);
      }
      qok = bar_and(2, 128, qok);
    } else if (!E8M0) {
      ts = *a.ts_x;   // written by the quantizer grid, complete since griddepcontrol.wait
    }
    if (tq == 0) {
      s_ts = ts;
      if (qok) mbar_arrive(xready);   // else the producer's bounded wait records the failure
      else s_fail = 1;
    }
    // the activation scales of every stage into TMEM (each warp its lane quadrant)
    const bool bok = __all_sync(0xFFFFFFFFu, mbar_wait(bfull, 0, 62));
    if (bok) {
      for (int it = 0; it < n_it; ++it)
        tmem_st_scale_atoms<Cfg::kAtoms>(tmem + quad_lanes + sfb_col(it), sSfb + it * Cfg::kSfBytes, lane);
      tmem_st_wait();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sfb_ok);
    if (!bok) s_fail = 1;
    if (!a.cluster && blockIdx.x == 0 && !amax_needed) {
      // CTA 0 advances the counter at its end: first every CTA's slot (each has read the counter)
      bool sok = true;
      for (int c = tq; c < G && sok; c += 128) dec_wait_tag(&sy.slots[c], tag, 54, sok);
      sok = bar_and(2, 128, sok);
      if (tq == 0) {
        s_allseen = sok ? 1 : 0;
        if (!sok) s_fail = 1;
      }
    }
    }   // cooperative / plain
  } else {
    if constexpr (VQ) {
      // ---------------- VQ decode (warps 2..9) into the ring of operand tiles: one warp
      // instruction covers 32 rows of one 32-element chunk (256 contiguous index bytes, lookups
      // in one 512-byte codebook, 16-byte stores hitting every bank once per 8 rows); warps 2..5
      // then put the stage's weight scales into their TMEM lane quadrant
      const int t = threadIdx.x - 64;
      for (int it = 0; it < n_it && ok; ++it) {
        const int slot = it % R;
        bool w = mbar_wait(&wfull[it], 0, 56);
        if (it >= R) w = w && mbar_wait(&aempty[slot], ((it / R) - 1) & 1, 57);
        if (!__all_sync(0xFFFFFFFFu, w)) { ok = false; break; }   // warp-uniform (tcgen05.st below)
        const uint8_t* idx_s = sW + it * Cfg::kWStride;
        const uint16_t* lut = reinterpret_cast<const uint16_t*>(idx_s + Cfg::kIdxBytes);
        uint8_t* a_s = sA + slot * Cfg::kABytes;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = t + 256 * j;
          const int kc = (c >> 5) & 7, r = (c & 31) | ((c >> 8) << 5);
          const uint2 iv = *reinterpret_cast<const uint2*>(idx_s + kc * 1024 + r * 8);
          const uint16_t* L = lut + ((((r >> 6) << 2) + (kc >> 1)) << 8);
          uint4 o;
          o.x = L[iv.x & 255u] | (static_cast<uint32_t>(L[(iv.x >> 8) & 255u]) << 16);
          o.y = L[(iv.x >> 16) & 255u] | (static_cast<uint32_t>(L[iv.x >> 24]) << 16);
          o.z = L[iv.y & 255u] | (static_cast<uint32_t>(L[(iv.y >> 8) & 255u]) << 16);
          o.w = L[(iv.y >> 16) & 255u] | (static_cast<uint32_t>(L[iv.y >> 24]) << 16);
          *reinterpret_cast<uint4*>(a_s + r * 128 + ((kc ^ (r & 7)) << 4)) = o;
        }
        fence_proxy_async_smem();
        if (warp < 6) {
          if constexpr (SF == 0) {
            tmem_st_scale_atoms<Cfg::kAtoms>(tmem + quad_lanes + sfa_col(it), idx_s + Cfg::kSfaOff, lane);
          } else {
            // lane i, column 4a + c: the 4 scales of row i + 32c in atom a (64 K = column QBlock
            // a): PostScale's one QBlock byte, or PreScale+'s codebook entry of group a / 2
            if (SF == 2 && it == 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(scbar, 0, 63)) && ok;
            const uint8_t* tail = idx_s + Cfg::kSfaOff;
            uint32_t v[16];
#pragma unroll
            for (int at = 0; at < 4; ++at)
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int r = lane + 32 * c;
                if constexpr (SF == 1) v[4 * at + c] = 0x01010101u * tail[(r >> 6) * 4 + at];
                else v[4 * at + c] = *reinterpret_cast<const uint32_t*>(sScb + tail[r * 2 + (at >> 1)] * 8 + (at & 1) * 4);
              }
            tmem_st16(tmem + quad_lanes + sfa_col(it), v);
          }
          tmem_st_wait();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&decd[slot]);
          if (warp < 6) mbar_arrive(&sfa_ok[it]);
        }
      }
    } else if (warp < 6) {
      // ---------------- the weight scales of every stage into TMEM as the blocks land
      for (int it = 0; it < n_it && ok; ++it) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&wfull[it], 0, 56))) { ok = false; break; }
        tmem_st_scale_atoms<Cfg::kAtoms>(tmem + quad_lanes + sfa_col(it), sW + it * Cfg::kWStride + Cfg::kSfaOff, lane);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfa_ok[it]);
      }
    }
    if (warp < 6) {
      // ---------------- epilogue: warps 2..5, TMEM lane quadrant = warp % 4
      const int q = warp & 3;
      const int nl = q * 32 + lane;
      const int n = n0 + nl;
      const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
      const int et = threadIdx.x - 64;   // 0..127
      // 8 accumulator columns from c: the odd stages' accumulator added when there were any
      auto ld_acc = [&](int c, uint32_t (&r)[8]) {
        tmem_ld8(trow + c, r);
        if (n_it > 1) {
          uint32_t r2[8];
          tmem_ld8(trow + BN + c, r2);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) r[jj] = __float_as_uint(__uint_as_float(r[jj]) + __uint_as_float(r2[jj]));
        } else {
          tmem_ld_wait();
        }
      };
      if (n_it > 0) ok = bar_and(1, 128, ok && mbar_wait(accf, 0, 58) && mbar_wait(xready, 0, 59));
      else ok = bar_and(1, 128, ok && mbar_wait(xready, 0, 59));
      tc_fence_after();
      float alpha = a.alpha;
      if (!E8M0) alpha *= s_ts;
      const uint32_t cnt = s_cnt;   // published before xready
      const unsigned long long tag = dec_tag(cnt + 1u);
      if (ok && a.splits == 1) {
#pragma unroll 1
        for (int c = 0; c < a.M; c += 8) {
          uint32_t r[8];
          ld_acc(c, r);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c + j < a.M && n < a.N) {
              const float v = (n_it > 0 ? __uint_as_float(r[j]) : 0.f) * alpha;
              const size_t o = static_cast<size_t>(c + j) * a.ldy + n;
              a.y[o] = __float2bfloat16_rn(v);
              if (a.y32 != nullptr) a.y32[o] = v;
            }
        }
      } else if (a.cluster) {
        // the partial [M][128] into this CTA's shared memory (the operand tiles are dead once
        // the accumulator is final), an arrival on every split's barrier, then this split's
        // share of the tile's outputs added over the splits in split order from their shared
        // memory (distributed shared memory loads)
        float* part = reinterpret_cast<float*>(smem);
        if (ok) {
#pragma unroll 1
          for (int c = 0; c < a.M; c += 8) {
            uint32_t r[8];
            ld_acc(c, r);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (c + j < a.M) part[(c + j) * 128 + nl] = n_it > 0 ? __uint_as_float(r[j]) : 0.f;
          }
        }
        named_bar_sync(1, 128);   // the whole partial is written before the releases
        if (et < S && !withheld(blockIdx.x)) mbar_arrive_remote(map_shared_rank(smem_u32(cpart), et));
        bool w = true;
        if (et == 0) w = mbar_wait_cluster(cpart, 0, 65);
        ok = bar_and(1, 128, ok && w);
        if (ok) {
          const int E4 = a.M * 32;
          const int q0 = static_cast<int>(static_cast<long>(E4) * z / S);
          const int q1 = static_cast<int>(static_cast<long>(E4) * (z + 1) / S);
          for (int qq = q0 + et; qq < q1; qq += 128) {
            const uint32_t la = smem_u32(part + (qq >> 5) * 128 + (qq & 31) * 4);
            float4 v[kDecMaxSplits];
#pragma unroll
            for (int r = 0; r < kDecMaxSplits; ++r)
              if (r < S) v[r] = ld_shared_cluster_f32x4(map_shared_rank(la, r));
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < kDecMaxSplits; ++r)
              if (r < S) {
                acc.x += v[r].x; acc.y += v[r].y; acc.z += v[r].z; acc.w += v[r].w;
              }
            dec_store4(a, qq >> 5, n0 + (qq & 31) * 4, acc, alpha);
          }
        }
      } else if (ok) {
        float* mine = a.partials + static_cast<size_t>(blockIdx.x) * BN * 128;
#pragma unroll 1
        for (int c = 0; c < a.M; c += 8) {
          uint32_t r[8];
          ld_acc(c, r);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c + j < a.M) mine[(c + j) * 128 + nl] = n_it > 0 ? __uint_as_float(r[j]) : 0.f;
        }
        named_bar_sync(1, 128);   // the whole partial is written before the release
        if (et == 0 && !withheld(blockIdx.x)) st_release_gpu_u64(&sy.pflags[blockIdx.x], tag | 1u);
        bool pok = true;
        if (et < a.splits) dec_wait_tag(&sy.pflags[tile * a.splits + et], tag, 60, pok);
        ok = bar_and(1, 128, pok);
        if (ok) {
          // this split's share of the tile's outputs in groups of 4 consecutive rows: every
          // split's partial loaded at once (16-byte loads through L2), then added in split order
          const int E4 = a.M * 32;                     // float4 groups of the tile
          const int q0 = static_cast<int>(static_cast<long>(E4) * z / a.splits);
          const int q1 = static_cast<int>(static_cast<long>(E4) * (z + 1) / a.splits);
          const float4* part0 = reinterpret_cast<const float4*>(a.partials) +
                                static_cast<size_t>(tile) * a.splits * BN * 32;
          for (int qq = q0 + et; qq < q1; qq += 128) {
            float4 v[kDecMaxSplits];
#pragma unroll
            for (int r = 0; r < kDecMaxSplits; ++r)
              if (r < a.splits) v[r] = __ldcg(part0 + static_cast<size_t>(r) * BN * 32 + qq);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < kDecMaxSplits; ++r)
              if (r < a.splits) {
                acc.x += v[r].x; acc.y += v[r].y; acc.z += v[r].z; acc.w += v[r].w;
              }
            dec_store4(a, qq >> 5, n0 + (qq & 31) * 4, acc, alpha);
          }
        }
      }
    }
  }
  if (!ok) s_fail = 1;
  tc_fence_before();
  if (a.cluster) cluster_sync_all();   // no CTA leaves while the others read its shared memory
  else __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
  // The next grid reads the counter only after this one has completed (griddepcontrol.wait).
  if (!a.cluster && threadIdx.x == 0) {
    if (s_fail) atomicAdd(sy.counter, 2u);
    else if (blockIdx.x == 0 && s_allseen) atomicAdd(sy.counter, 1u);
  }
}

}  // namespace ql
