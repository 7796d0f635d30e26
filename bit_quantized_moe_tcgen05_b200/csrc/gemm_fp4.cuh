// Block-scaled FP4 GEMM on tcgen05 tensor cores (sm_100a), with the PRQuant K-extension.
//
//   y[m, n] = alpha * sum_k x_q[m, k] * w_q[n, k]
//
// over packed E2M1 operands with per-32 E8M0 scales (kind::mxf4) or per-16 UE4M3 scales
// (kind::mxf4nvf4, alpha = product of the two FP32 tensor scales).  The weight is the MMA's
// 128-row "A" operand and the tokens are the "B" operand of width BN (16..256), so one kernel
// serves decode (M = 1..64, with split-K over CTAs) and prefill (M up to thousands).
//
// PRQuant ("Kernel design for efficient inference"): the weight is W_aug = Q([W~, R_W]) with
// reduction width C + k; the activation is quantized once over its C channels and its last k
// channels are read a second time for the tail stages (activation coordinate C - k + j while
// the weight coordinate is C + j).  No tail copy is materialised.
//
// Warp roles (192 threads; 352 for VQ weights): warp 0 = TMA producer, warp 1 = TMEM allocator +
// MMA issuer (one lane issues), warps 2..5 = epilogue; with VQ weights warps 2..9 first rebuild
// each stage's operand tile from the codebooks.  Where TMEM holds two accumulators, a second warp
// (warp 2, or warp 10 with VQ) issues the MMAs of every other stage into the second one (the
// epilogue adds the two); without VQ, warp 3 produces every other stage.  A STAGES-deep ring of
// shared-memory stages, each 256 K-elements deep, is guarded by full/empty mbarriers; MMA
// completion is signalled by tcgen05.commit.  Every wait is bounded (see ptx.cuh).
//
// Weight streaming starts before the activations exist: the kernel is launched with programmatic
// stream serialization behind the activation quantizer, the producer first issues the weight
// copies of the whole first ring fill (and the VQ warps decode them), and only then waits for the
// quantizer grid (griddepcontrol.wait) before it loads activation tiles.  In decode launches the
// activation tiles and scale atoms of every stage go by cp.async from the producer warp, so they
// do not queue behind the weight blocks in the bulk-copy engine.  Every CTA also releases the
// next programmatic grid at once (griddepcontrol.launch_dependents): the next layer's quantizer
// and GEMM then take SMs as this grid's CTAs retire and start their weight streams during this
// grid's split-K tail.  Whatever they read of this grid's results (y, the workspace) they read
// after their own griddepcontrol.wait, which returns only once this grid has completed.
//
// Work: a 1-D grid.  Tiles (128 weight rows x BN tokens, weight tile fastest) [0, full_tiles) get
// one CTA each over all K; the remaining tiles are split along K over `splits` CTAs each.
// Decode launches split every tile (full_tiles = 0) so that the grid covers the SMs; launches with
// at least a wave of tiles run them all unsplit (the kernel also accepts whole tiles followed by
// split ones, which measured slower for the leftover tiles of the last wave).  The K-splits
// of a tile each write an fp32 partial tile to a global workspace; the last split to finish (an
// atomic ticket per tile) bulk-copies the partials into its idle ring and adds them in split
// order, so the result is deterministic, writes y and re-arms the ticket.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace ql {

// Most K-splits of one output tile (bounds the per-thread partial loads of the reduction).
constexpr int kMaxSplits = 8;

struct Fp4GemmArgs {
  int M, N;                 // tokens, output features
  int C, k_tail;            // activation width; tail width (weight width K' = C + k_tail)
  int n_base_stages;        // ceil(C / 256)
  int n_stages_total;       // n_base_stages + ceil(k_tail / 256)
  int stages_per_split;     // K stages handled by one CTA of a split tile
  int tiles_n;              // 128-row weight tiles
  int full_tiles;           // tiles [0, full_tiles) are not split
  int splits;               // K-splits of every other tile
  const uint8_t* sfb;       // activation scales, tiled atoms
  int sfb_atoms;            // atoms per 128-row group of the activation
  const float* alpha_dev;   // optional device scalar multiplied into alpha (tensor scale of x)
  float alpha;              // host scalar (tensor scale of w, or 1)
  __nv_bfloat16* y;         // [M, ldy] bf16 output
  float* y32;               // optional [M, ldy] fp32 output
  int ldy;
  const uint8_t* wt;        // weight blocks [N/128][n_stages_total][Fp4Cfg::kWBytes], one per
                            // (128-row tile, 256-wide K stage), laid out as the stage buffer:
                            // FP4 codes 128 rows x 128 B with the 128-byte swizzle applied, or VQ
                            // indices 128 rows x 64 B + the stage's 8 QBlock codebooks; then the
                            // stage's weight scale atoms
  float* partials;          // split tiles: fp32 [tile - full_tiles][splits][BN][128]
  const uint8_t* xq;        // quantized activation codes [M, C/2] (read directly by decode launches)
  int* tickets;             // [split tiles] arrival counters, zero between launches
  const uint8_t* scb;       // VQ PreScale+: scale codebook [256][8] E4M3 bytes
  int act_aug;              // the quantized activation is already augmented ([M, C + k_tail]:
                            // the tail copied behind, PRQuant's offline copy): tail stages read
                            // activation coordinate C + j, like the weight
};

// SF (VQ weights only): where the weight's E4M3 block scales come from -- 0 MXCode PreScale (the
// stage's scale atoms are stored in its block), 1 PostScale (one scale per 64 x 64 QBlock: the
// block ends with the stage's 8 QBlock bytes), 2 PreScale+ (the block ends with 2 scale indices
// per row into a 256 x 8 scale codebook).  For 1 and 2 the decoders build the scale atoms.
template <int BN, bool E8M0, bool VQ = false, int SF = 0>
struct Fp4Cfg {
  // warps: 0 producer, 1 MMA, 2..5 epilogue; VQ adds decoders so that warps 2..9 decode
  static constexpr int kDecWarps = VQ ? 8 : 0;
  static constexpr int kThreads = VQ ? 352 : 192;   // VQ: warp 10 is the second MMA issuer
  static constexpr int kAtomK = E8M0 ? 128 : 64;      // K elements covered by one SF atom
  static constexpr int kAtoms = 256 / kAtomK;         // SF atoms per stage per 128 rows
  static constexpr int kG = (BN + 127) / 128;          // 128-row groups of the B operand
  static constexpr int kABytes = 128 * 128;            // 128 rows x 256 fp4
  static constexpr int kBBytes = BN * 128;
  static constexpr int kSfaBytes = kAtoms * 512;
  static constexpr int kSfbBytes = kAtoms * kG * 512;
  static constexpr int kIdxBytes = VQ ? 128 * 64 : 0;   // VQ: 8-bit indices [chunk 8][row 128][8]
  static constexpr int kLutBytes = VQ ? 8 * 512 : 0;    // VQ: 2 x 4 QBlock codebooks of 512 B
  // The weight block of one stage, as stored in HBM and copied by one bulk copy:
  // FP4: [codes 16 KB][SFA atoms]; VQ: [indices 8 KB, chunk-major][codebooks 4 KB][SFA atoms].
  static_assert(SF == 0 || (VQ && !E8M0), "PostScale / PreScale+ scales: VQ E4M3-B16 weights");
  static constexpr int kSfTail = SF == 0 ? kSfaBytes : SF == 1 ? 16 : 256;
  static constexpr int kWBytes = (VQ ? kIdxBytes + kLutBytes : kABytes) + kSfTail;   // in HBM
  static constexpr int kWStride = (kWBytes + 1023) / 1024 * 1024;                     // in smem
  static constexpr int kSfaOff = VQ ? kIdxBytes + kLutBytes : kABytes;
  static constexpr int kSfaBuild = SF != 0 ? kSfaBytes : 0;   // built scale atoms per stage
  static constexpr int kScbBytes = SF == 2 ? 2048 : 0;        // PreScale+ scale codebook
  static constexpr int kStageBytes = kWStride + kBBytes + kSfbBytes + (VQ ? kABytes : 0) + kSfaBuild;
  static constexpr int kBudget = 212 * 1024;
  static constexpr int kStagesRaw = kBudget / kStageBytes;
  static constexpr int kStages = kStagesRaw > 12 ? 12 : (kStagesRaw < 2 ? 2 : kStagesRaw);
  static constexpr int kSfaCols = kAtoms * 4;          // TMEM columns per stage
  static constexpr int kSfbCols = kAtoms * 4 * kG;
  // Where TMEM holds two accumulators a second warp (without VQ the first epilogue warp, idle
  // during the main loop; with VQ an extra warp) issues the MMAs of every other stage into the
  // second one: issuing a block-scaled MMA and its scale copies costs the issuing thread more
  // than the tensor core needs to run it.
  static constexpr int kIssuers = (2 * BN + kStages * (kSfaCols + kSfbCols) <= 512) ? 2 : 1;
  static constexpr int kIssuer2Warp = VQ ? 10 : 2;
  static constexpr int kColsNeeded = kIssuers * BN + kStages * (kSfaCols + kSfbCols);
  static constexpr int kProducers = VQ ? 1 : 2;   // without VQ, warp 3 also produces
  static constexpr int kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64
                                 : kColsNeeded <= 128 ? 128 : kColsNeeded <= 256 ? 256 : 512;
  static_assert(kColsNeeded <= 512, "TMEM budget");
  static constexpr int kSmemBytes = kStages * kStageBytes + kScbBytes + 1024 /*align*/ + 512 /*barriers*/;
  static_assert(BN * 128 * 4 <= kStages * kStageBytes, "output staging must fit the ring");
};

// The weight operand of each (128-row tile, K stage) is one contiguous block in HBM, laid out at
// create time exactly as the stage buffer wants it, and arrives by one 1-D bulk copy.
// VQ = true (MXCode PreScale weights): the blocks hold 8-bit indices; warps 2..9 decode each
// stage's operand tile from the shared-memory codebooks.
template <int BN, bool E8M0, bool VQ = false, int SF = 0>
__global__ void __launch_bounds__(Fp4Cfg<BN, E8M0, VQ, SF>::kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
                    const __grid_constant__ CUtensorMap tm_y32, const Fp4GemmArgs a) {
  using Cfg = Fp4Cfg<BN, E8M0, VQ, SF>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  // 1 KB aligned by offsetting the shared array itself, so that every pointer derived from it
  // stays a shared-space pointer (plain ld/st.shared, not generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  // ring layout (every region 1 KB aligned): weight blocks, B tiles, SFB atoms, decoded A (VQ)
  uint8_t* sW = smem;
  uint8_t* sB = sW + S * Cfg::kWStride;
  uint8_t* sSfb = sB + S * Cfg::kBBytes;
  uint8_t* sAdec = sSfb + S * Cfg::kSfbBytes;
  auto sA = [&](int st) { return VQ ? sAdec + st * Cfg::kABytes : sW + st * Cfg::kWStride; };
  uint8_t* sSfaB = sAdec + (VQ ? S * Cfg::kABytes : 0);   // SF 1/2: the stages' built scale atoms
  uint8_t* sScb = sSfaB + S * Cfg::kSfaBuild;              // SF 2: the scale codebook
  uint64_t* full = reinterpret_cast<uint64_t*>(sScb + Cfg::kScbBytes);
  uint64_t* empty = full + S;
  uint64_t* decd = empty + S;   // VQ: operand tile decoded
  uint64_t* wfull = decd + S;   // VQ: indices + codebooks + SFA landed
  uint64_t* afull = wfull + S;  // decode: activation tile + SFB landed by cp.async (count 32)
  uint64_t* accf = afull + S;   // accumulator complete
  uint64_t* rbar = accf + 1;    // split-K: the splits' partials landed in the idle ring
  uint64_t* scbar = rbar + 1;   // SF 2: the scale codebook landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(scbar + 1);
  __shared__ int s_last;
  griddep_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int tile, zsplit, splits;
  if (static_cast<int>(blockIdx.x) < a.full_tiles) {
    tile = blockIdx.x;
    zsplit = 0;
    splits = 1;
  } else {
    const int r = blockIdx.x - a.full_tiles;
    tile = a.full_tiles + r / a.splits;
    zsplit = r % a.splits;
    splits = a.splits;
  }
  const int wtile = tile % a.tiles_n;
  const int n0 = wtile * 128, m0 = (tile / a.tiles_n) * BN;
  const int sf_group0 = (tile / a.tiles_n) * Cfg::kG;   // first 128-row scale group of the tile
  const int s_begin = splits == 1 ? 0 : zsplit * a.stages_per_split;
  const int s_end = splits == 1 ? a.n_stages_total : min(a.n_stages_total, s_begin + a.stages_per_split);
  const int n_it = max(0, s_end - s_begin);
  // decode launches whose stages all fit the ring take activations by cp.async
  const bool lsu_act = BN <= 64 && n_it <= S;

  // K stage i -> (weight element offset, activation element offset, valid elements)
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
  // Weight part of stage it (independent of earlier grids): one bulk copy of the stage block.
  auto issue_weight = [&](int it) {
    const int i = s_begin + it, st = it % S;
    int kw, kx, valid;
    stage_coords(i, kw, kx, valid);
    const int nat = valid / Cfg::kAtomK;
    const uint32_t act_bytes = lsu_act ? 0u : Cfg::kBBytes + nat * 512 * Cfg::kG;
    const uint8_t* wblk = a.wt + (static_cast<size_t>(wtile) * a.n_stages_total + i) * Cfg::kWBytes;
    if constexpr (VQ) {
      mbar_arrive_expect_tx(&wfull[st], Cfg::kWBytes);
      if (!lsu_act) mbar_arrive_expect_tx(&full[st], act_bytes);
      bulk_load(sW + st * Cfg::kWStride, wblk, Cfg::kWBytes, &wfull[st]);
    } else {
      mbar_arrive_expect_tx(&full[st], Cfg::kWBytes + act_bytes);
      bulk_load(sW + st * Cfg::kWStride, wblk, Cfg::kWBytes, &full[st]);
    }
  };
  const int pre = min(n_it, S);   // the first ring fill needs no empty-slot wait

  // Warp 0 initialises the barriers (lane s: stage s) and, before the block-wide barrier, its lane
  // 0 already issues the weight copies of the first ring fill, so that they are in flight while
  // the TMEM allocation and the rest of the set-up run.
  if (warp == 0) {
    for (int s = lane; s < S; s += 32) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&decd[s], VQ ? Cfg::kDecWarps : 1);
      mbar_init(&wfull[s], 1);
      mbar_init(&afull[s], 32);
    }
    if (lane == 0) {
      mbar_init(accf, Cfg::kIssuers);
      mbar_init(rbar, 1);
      mbar_init(scbar, 1);
    }
    fence_mbar_init();
    __syncwarp();
    if (lane == 0) {
      if constexpr (SF == 2) {
        mbar_arrive_expect_tx(scbar, Cfg::kScbBytes);
        bulk_load(sScb, a.scb, Cfg::kScbBytes, scbar);
      }
      for (int it = 0; it < pre; ++it) issue_weight(it);
      prefetch_tmap(&tm_x);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sfa_col0 = Cfg::kIssuers * BN, sfb_col0 = Cfg::kIssuers * BN + S * Cfg::kSfaCols;

  bool ok = true;
  // ---------------- MMA issuer j (converged warp, one lane issues the tcgen05 instructions):
  // stages j, j + kIssuers, ... into accumulator j
  auto mma_issue = [&](int j) {
    const uint32_t idesc0 = idesc_fp4_block(BN, E8M0);
    const uint32_t dacc = tmem + j * BN;
    for (int it = j; it < n_it && ok; it += Cfg::kIssuers) {
      const int i = s_begin + it, st = it % S;
      const uint32_t ph = (it / S) & 1;
      bool w = true;
      if (!VQ || !lsu_act) w = mbar_wait(&full[st], ph, 2);
      if constexpr (VQ) w = w && mbar_wait(&wfull[st], ph, 6) && mbar_wait(&decd[st], ph, 4);
      if (lsu_act) w = w && mbar_wait(&afull[st], 0, 9);
      ok = __all_sync(0xFFFFFFFFu, w);
      if (!ok) break;
      tc_fence_after();
      int kw, kx, valid;
      stage_coords(i, kw, kx, valid);
      const int nat = valid / Cfg::kAtomK;
      const uint32_t ta = tmem + sfa_col0 + st * Cfg::kSfaCols;
      const uint32_t tb = tmem + sfb_col0 + st * Cfg::kSfbCols;
      const uint32_t sfa_s = SF != 0 ? smem_u32(sSfaB + st * Cfg::kSfaBuild)
                                     : smem_u32(sW + st * Cfg::kWStride + Cfg::kSfaOff);
      const uint32_t sfb_s = smem_u32(sSfb + st * Cfg::kSfbBytes);
      const uint32_t a_base = smem_u32(sA(st));
      const uint32_t b_base = smem_u32(sB + st * Cfg::kBBytes);
      const int nk = valid / 64;
      if (lane == 0) {   // the same lane issues every MMA and the commits that track them
#pragma unroll
        for (int at = 0; at < Cfg::kAtoms; ++at) {
          if (at < nat) {
            tc_cp_32x128b_warpx4(ta + at * 4, make_sdesc(sfa_s + at * 512, 0, 128, kLayoutNone));
#pragma unroll
            for (int gg = 0; gg < Cfg::kG; ++gg)
              tc_cp_32x128b_warpx4(tb + at * 4 * Cfg::kG + gg * 4,
                                   make_sdesc(sfb_s + gg * Cfg::kAtoms * 512 + at * 512, 0, 128, kLayoutNone));
          }
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          if (kk < nk) {
            const int at = (kk * 64) / Cfg::kAtomK;
            const uint32_t byte = E8M0 ? static_cast<uint32_t>((kk & 1) * 2) : 0u;
            const uint64_t ad = make_sdesc(a_base + kk * 32, 16, 1024, kLayoutSW128);
            const uint64_t bd = make_sdesc(b_base + kk * 32, 16, 1024, kLayoutSW128);
            const uint32_t idd = idesc0 | (byte << 29) | (byte << 4);
            const uint32_t sa = (ta + at * 4) | (byte << 30);
            const uint32_t sb = (tb + at * 4 * Cfg::kG) | (byte << 30);
            const uint32_t acc = (it == j && kk == 0) ? 0u : 1u;
            if (E8M0)
              mma_mxf4_block32(dacc, ad, bd, idd, sa, sb, acc);
            else
              mma_nvf4_block16(dacc, ad, bd, idd, sa, sb, acc);
          }
        }
        tc_commit(&empty[st]);
      }
      __syncwarp();
    }
    if (lane == 0) tc_commit(accf);
    __syncwarp();
  };
  // ---------------- producer: the whole warp runs the loop; one elected lane issues copies.
  // Activation part (written by the quantizer grid): B codes and SFB, by the bulk-copy engine.
  auto issue_act = [&](int it) {
    const int i = s_begin + it, st = it % S;
    int kw, kx, valid;
    stage_coords(i, kw, kx, valid);
    if (a.act_aug) kx = kw;
    const int nat = valid / Cfg::kAtomK;
    tma_load_2d(sB + st * Cfg::kBBytes, &tm_x, &full[st], kx >> 1, m0);
#pragma unroll
    for (int g = 0; g < Cfg::kG; ++g)
      bulk_load(sSfb + st * Cfg::kSfbBytes + g * Cfg::kAtoms * 512,
                a.sfb + (static_cast<size_t>(sf_group0 + g) * a.sfb_atoms + kx / Cfg::kAtomK) * 512,
                nat * 512, &full[st]);
  };
  // Steady state of the ring from stage `pre` on: producer j takes the stages of parity j (two
  // producers without VQ: a stage's empty-slot wait and its copies cost the issuing thread
  // about as long as the tensor core needs for the stage).
  auto produce = [&](int j) {
    for (int it = pre; it < n_it && ok; ++it) {
      if (Cfg::kProducers == 2 && (it & 1) != j) continue;
      const int st = it % S;
      const uint32_t ph = (it / S) & 1;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&empty[st], ph ^ 1, 1));
      if (!ok) break;
      if (elect_one()) {
        issue_weight(it);
        issue_act(it);
      }
      __syncwarp();
    }
  };
  if (warp == 0) {
    griddep_wait();
    if (lsu_act) {
      // Every stage's activation tile (BN rows x 128 B, stored with the 128-byte swizzle) and its
      // scale atoms, 16 bytes per cp.async from all 32 lanes; rows past M are zero-filled.
      const int xw2 = (a.act_aug ? a.C + a.k_tail : a.C) / 2;   // bytes per activation row
      for (int it = 0; it < n_it; ++it) {
        int kw, kx, valid;
        stage_coords(s_begin + it, kw, kx, valid);
        if (a.act_aug) kx = kw;
        const int nat = valid / Cfg::kAtomK;
        const uint32_t bdst = smem_u32(sB + it * Cfg::kBBytes);
        for (int c = lane; c < BN * 8; c += 32) {
          const int r = c >> 3, kc = c & 7;
          const bool in = m0 + r < a.M;
          const uint8_t* src = a.xq + static_cast<size_t>(in ? m0 + r : 0) * xw2 + (kx >> 1) + kc * 16;
          cp_async16(bdst + r * 128 + ((kc ^ (r & 7)) << 4), src, in ? 16u : 0u);
        }
        const uint8_t* sfsrc = a.sfb + (static_cast<size_t>(sf_group0) * a.sfb_atoms + kx / Cfg::kAtomK) * 512;
        const uint32_t sfdst = smem_u32(sSfb + it * Cfg::kSfbBytes);
        for (int c = lane; c < nat * 32; c += 32) cp_async16(sfdst + c * 16, sfsrc + c * 16, 16u);
        cp_async_commit();
      }
      for (int it = 0; it < n_it; ++it) {   // stage it complete -> visible to the tensor core
        cp_async_wait_pending(n_it - 1 - it);
        fence_proxy_async_smem();
        mbar_arrive(&afull[it]);
      }
    } else {
      if (elect_one())
        for (int it = 0; it < pre; ++it) issue_act(it);
      __syncwarp();
      produce(0);
    }
  } else if (warp == 1) {
    mma_issue(0);
  } else if (VQ && warp == Cfg::kIssuer2Warp) {
    if (Cfg::kIssuers == 2) mma_issue(1);
  } else {
    if constexpr (VQ) {
      // ---------------- VQ decode (warps 2..9): for each stage rebuild the 128 x 256 E2M1 operand
      // tile from 8-bit indices and the QBlock codebooks, in the 128-byte-swizzled K-major layout
      // the MMA reads (16-byte chunk kc of row r at kc ^ (r%8)).  Only weights are read, so this
      // runs ahead of the activation quantizer.  One warp instruction covers 32 consecutive rows
      // of one 32-element chunk: its index loads are 256 contiguous bytes (the block stores the
      // indices chunk-major), its lookups all fall in one 512-byte codebook, and its 16-byte
      // stores hit every bank once per 8 rows.
      const int t = threadIdx.x - 64;
      constexpr int kDT = Cfg::kDecWarps * 32;
      static_assert(1024 % kDT == 0 && kDT % 256 == 0, "decoder threads tile the 1024 chunks");
      for (int it = 0; it < n_it && ok; ++it) {
        const int st = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!mbar_wait(&wfull[st], ph, 5)) { ok = false; break; }
        const uint8_t* idx_s = sW + st * Cfg::kWStride;
        const uint16_t* lut = reinterpret_cast<const uint16_t*>(idx_s + Cfg::kIdxBytes);
        uint8_t* a_s = sA(st);
#pragma unroll
        for (int j = 0; j < 1024 / kDT; ++j) {
          const int c = t + kDT * j;
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
        if constexpr (SF != 0) {
          // the stage's four scale atoms (row r at (r%32)*16 + ((r/32)%4)*4, 4 scale columns per
          // atom): PostScale gives all 16-blocks of a QBlock its one byte, PreScale+ looks the
          // row's two 8-scale groups up in the scale codebook
          if (SF == 2 && it == 0 && !mbar_wait(scbar, 0, 7)) { ok = false; }
          const uint8_t* tail = idx_s + Cfg::kSfaOff;
          uint8_t* sfa = sSfaB + st * Cfg::kSfaBuild;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int wi = t + kDT * j;          // 512 words: atom wi / 128, row wi % 128
            if (wi < 512) {
              const int at = wi >> 7, r = wi & 127;
              uint32_t word;
              if constexpr (SF == 1) word = 0x01010101u * tail[(r >> 6) * 4 + at];
              else word = *reinterpret_cast<const uint32_t*>(sScb + tail[r * 2 + (at >> 1)] * 8 + (at & 1) * 4);
              *reinterpret_cast<uint32_t*>(sfa + at * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4) = word;
            }
          }
        }
        fence_proxy_async_smem();   // every writer orders its stores for the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&decd[st]);
      }
    }
    if (!VQ && Cfg::kIssuers == 2 && warp == Cfg::kIssuer2Warp) mma_issue(1);
    if (Cfg::kProducers == 2 && warp == 3 && !lsu_act) {
      griddep_wait();   // the activations of this grid's quantizer
      produce(1);
    }
    if (warp < 6) {   // (extra VQ decoders, warps 6..9, take no part in the epilogue)
      // ---------------- epilogue: warps 2..5, TMEM lane quadrant = warp % 4
      const int q = warp & 3;
      const int nl = q * 32 + lane;
      const int n = n0 + nl;
      const int mcount = min(BN, a.M - m0);
      const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
      // 8 accumulator columns from c: the second issuer's accumulator added when it ran a stage
      const bool two = Cfg::kIssuers == 2 && n_it > 1;
      auto ld_acc = [&](int c, uint32_t (&r)[8]) {
        tmem_ld8(trow + c, r);
        if (two) {
          uint32_t r2[8];
          tmem_ld8(trow + BN + c, r2);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) r[jj] = __float_as_uint(__uint_as_float(r[jj]) + __uint_as_float(r2[jj]));
        } else {
          tmem_ld_wait();
        }
      };
      // Unsplit epilogue: kEc columns from c with every TMEM load of both accumulators in flight
      // before one wait (a wait per 8 columns serialised the load latency: 41.0 -> 38.9 us at
      // 2048 tokens). The VQ instantiations keep the 8-column loads.
      constexpr int kEc = VQ ? 8 : (BN % 32 == 0 ? 32 : (BN % 16 == 0 ? 16 : 8));
      auto ld_accn = [&](int c, uint32_t (&r)[kEc]) {
#pragma unroll
        for (int e = 0; e < kEc; e += 8) tmem_ld8(trow + c + e, *reinterpret_cast<uint32_t(*)[8]>(r + e));
        if (two) {
          uint32_t r2[kEc];
#pragma unroll
          for (int e = 0; e < kEc; e += 8) tmem_ld8(trow + BN + c + e, *reinterpret_cast<uint32_t(*)[8]>(r2 + e));
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < kEc; ++jj) r[jj] = __float_as_uint(__uint_as_float(r[jj]) + __uint_as_float(r2[jj]));
        } else {
          tmem_ld_wait();
        }
      };
      griddep_wait();   // alpha_dev, the workspace and y belong to / follow earlier grids
      float alpha = a.alpha;
      if (a.alpha_dev != nullptr) alpha *= *a.alpha_dev;
      if (n_it > 0) ok = bar_and(1, 128, ok && mbar_wait(accf, 0, 3));   // the 128 agree
      tc_fence_after();
      if (ok && splits == 1) {
        // The tile is staged in the idle operand ring as y[m][n] and written by one TMA tensor
        // store (which clips rows past M and columns past N): first the bf16 tile, then, when
        // requested, the fp32 tile in the same buffer once the first store has read it.
        __nv_bfloat16* ybuf = reinterpret_cast<__nv_bfloat16*>(smem);               // [BN][128]
        float* y32buf = reinterpret_cast<float*>(smem);                             // [BN][128]
#pragma unroll 1
        for (int c = 0; c < BN; c += kEc) {
          uint32_t r[kEc];
          if constexpr (VQ) ld_acc(c, r); else ld_accn(c, r);
#pragma unroll
          for (int j = 0; j < kEc; ++j)
            ybuf[(c + j) * 128 + nl] = __float2bfloat16_rn((n_it > 0 ? __uint_as_float(r[j]) : 0.f) * alpha);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) {
          tma_store_2d(&tm_y, ybuf, n0, m0);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
        if (a.y32 != nullptr) {
          named_bar_sync(1, 128);
#pragma unroll 1
          for (int c = 0; c < BN; c += kEc) {
            uint32_t r[kEc];
            if constexpr (VQ) ld_acc(c, r); else ld_accn(c, r);
#pragma unroll
            for (int j = 0; j < kEc; ++j) y32buf[(c + j) * 128 + nl] = (n_it > 0 ? __uint_as_float(r[j]) : 0.f) * alpha;
          }
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (threadIdx.x == 64) {
            tma_store_2d(&tm_y32, y32buf, n0, m0);
            bulk_commit_group();
            bulk_wait_group_read0();
          }
        }
      } else if (ok) {
        // Split-K: park this split's fp32 partial [BN tokens][128 rows] in the workspace (lanes
        // cover consecutive rows: coalesced) and take a ticket; the last split reduces.
        const int stile = tile - a.full_tiles;   // index among the split tiles
        float* part = a.partials + static_cast<size_t>(stile) * splits * BN * 128;
        float* mine = part + static_cast<size_t>(zsplit) * BN * 128;
#pragma unroll 1
        for (int c = 0; c < mcount; c += 8) {
          uint32_t r[8];
          ld_acc(c, r);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c + j < mcount) mine[(c + j) * 128 + nl] = n_it > 0 ? __uint_as_float(r[j]) : 0.f;
        }
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) {
          // releases the whole CTA's partial (ordered before by the barrier); the last split
          // acquires every other split's
          s_last = atom_add_acq_rel_gpu(reinterpret_cast<uint32_t*>(a.tickets + stile), 1u) ==
                   static_cast<uint32_t>(splits - 1);
        }
        named_bar_sync(1, 128);
        if (s_last) {
          // The ring is idle: bulk-copy every split's partial for a run of tokens into it (all
          // copies in flight at once), then each thread adds its row in split order, 4 tokens at
          // a time with every split's value of them loaded before the adds.
          float* stg = reinterpret_cast<float*>(smem);
          constexpr int kRing = S * Cfg::kStageBytes;
          const int cc = min(mcount, (kRing / (splits * 512)) & ~7);
#pragma unroll 1
          for (int c0 = 0, rnd = 0; c0 < mcount && ok; c0 += cc, ++rnd) {
            const int cn = min(cc, mcount - c0);
            if (threadIdx.x == 64) {
              fence_proxy_async_global();
              mbar_arrive_expect_tx(rbar, splits * cn * 512);
              for (int r = 0; r < splits; ++r)
                bulk_load(stg + r * cc * 128, part + (static_cast<size_t>(r) * BN + c0) * 128, cn * 512, rbar);
            }
            ok = bar_and(1, 128, mbar_wait(rbar, rnd & 1, 8));
            if (!ok) break;
#pragma unroll 1
            for (int c = 0; c < cn; c += 4) {
              float v[kMaxSplits][4];
#pragma unroll
              for (int r = 0; r < kMaxSplits; ++r)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  v[r][j] = (r < splits && c + j < cn) ? stg[(r * cc + c + j) * 128 + nl] : 0.f;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                float acc = 0.f;
#pragma unroll
                for (int r = 0; r < kMaxSplits; ++r)
                  if (r < splits) acc += v[r][j];
                if (c + j < cn && n < a.N) {
                  const size_t o = static_cast<size_t>(m0 + c0 + c + j) * a.ldy + n;
                  a.y[o] = __float2bfloat16_rn(acc * alpha);
                  if (a.y32 != nullptr) a.y32[o] = acc * alpha;
                }
              }
            }
            named_bar_sync(1, 128);   // before the next run overwrites stg
          }
          if (threadIdx.x == 64) a.tickets[stile] = 0;   // re-armed for the next launch
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace ql
