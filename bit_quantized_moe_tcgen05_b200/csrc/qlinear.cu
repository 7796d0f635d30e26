// libqlinear: C ABI over the sm_100a kernels (see include/qlinear.h for the contract).
// One translation unit holds every kernel so that they share the device error word.
#include "qlinear.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "ptx.cuh"
#include "quant_act.cuh"
#include "gemm_fp4.cuh"
#include "decode_fp4.cuh"
#include "moe.cuh"
#include "int4_gemm.cuh"
#include "peak.cuh"

namespace {

thread_local std::string g_last_error;

ql_status fail(ql_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define QL_CUDA(call)                                                                  \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess)                                                             \
      return fail(QL_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));        \
  } while (0)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ----------------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D byte tensor [rows, inner_bytes], box [box_rows, box_inner bytes], 128-byte swizzle unless
// `swizzle` is false.
ql_status make_tmap_u8(CUtensorMap* m, const void* base, uint64_t inner_bytes, uint64_t rows,
                       uint64_t row_stride, uint32_t box_inner, uint32_t box_rows,
                       bool swizzle = true) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(QL_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner_bytes, rows};
  cuuint64_t strides[1] = {row_stride};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return QL_OK;
}

// 2-D bf16 tensor [rows, cols] with a 128-byte swizzled box [box_rows, 64 elements].
ql_status make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                         uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(QL_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QL_ERR_CUDA, "cuTensorMapEncodeTiled (bf16) failed (%d)", int(r));
  return QL_OK;
}

// Output tensor [rows, cols] (bf16 or fp32, row-major, no swizzle), box [box_rows, 128 cols].
ql_status make_tmap_out(CUtensorMap* m, const void* base, bool f32, uint64_t cols, uint64_t rows,
                        uint64_t ld, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(QL_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * es};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QL_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", int(r));
  return QL_OK;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// ----------------------------------------------------------------------- GEMM launch
// The GEMM is launched with programmatic stream serialization: it may start while the kernel
// before it on the stream (the activation quantizer) is still running, and streams (and, for VQ,
// decodes) weights until its griddepcontrol.wait.
template <int BN, bool E8M0, bool VQ, int SF = 0>
ql_status launch_fp4_bn(const CUtensorMap& tx, const CUtensorMap& ty, const CUtensorMap& ty32,
                        const ql::Fp4GemmArgs& a, dim3 grid, cudaStream_t s) {
  using Cfg = ql::Fp4Cfg<BN, E8M0, VQ, SF>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    QL_CUDA(cudaFuncSetAttribute(ql::fp4_gemm_kernel<BN, E8M0, VQ, SF>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
    attr_done[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  QL_CUDA(cudaLaunchKernelEx(&cfg, ql::fp4_gemm_kernel<BN, E8M0, VQ, SF>, tx, ty, ty32, a));
  return QL_OK;
}

template <bool E8M0, bool VQ, int SF = 0>
ql_status launch_fp4(int BN, const CUtensorMap& tx, const CUtensorMap& ty, const CUtensorMap& ty32,
                     const ql::Fp4GemmArgs& a, dim3 grid, cudaStream_t s) {
  switch (BN) {
    case 16: return launch_fp4_bn<16, E8M0, VQ, SF>(tx, ty, ty32, a, grid, s);
    case 32: return launch_fp4_bn<32, E8M0, VQ, SF>(tx, ty, ty32, a, grid, s);
    case 64: return launch_fp4_bn<64, E8M0, VQ, SF>(tx, ty, ty32, a, grid, s);
    case 128: return launch_fp4_bn<128, E8M0, VQ, SF>(tx, ty, ty32, a, grid, s);
    case 160: return launch_fp4_bn<160, E8M0, VQ, SF>(tx, ty, ty32, a, grid, s);
    case 256: return launch_fp4_bn<256, E8M0, VQ, SF>(tx, ty, ty32, a, grid, s);
  }
  return fail(QL_ERR_UNSUPPORTED, "no GEMM tile for BN=%d", BN);
}

// The decode kernel's launch attributes, set once per device (dynamic shared memory above 48 KB;
// clusters of up to 16 CTAs).
template <int BN, bool E8M0, bool VQ, int SF = 0>
ql_status dec_set_attrs() {
  using Cfg = ql::DecCfg<BN, E8M0, VQ, SF>;
  static std::atomic<bool> attr_done[64] = {};
  int dev = 0;
  QL_CUDA(cudaGetDevice(&dev));
  if (dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
    QL_CUDA(cudaFuncSetAttribute(ql::fp4_decode_kernel<BN, E8M0, VQ, SF>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
    QL_CUDA(cudaFuncSetAttribute(ql::fp4_decode_kernel<BN, E8M0, VQ, SF>,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    if (dev < 64) attr_done[dev].store(true, std::memory_order_release);
  }
  return QL_OK;
}

// How many clusters of S decode CTAs the device can hold at once (0 if none), cached per
// (device, S).
template <int BN, bool E8M0, bool VQ, int SF = 0>
int dec_max_clusters_bn(int S) {
  using Cfg = ql::DecCfg<BN, E8M0, VQ, SF>;
  static std::atomic<int> cache[64][ql::kDecMaxSplits + 1];
  static std::atomic<bool> known[64][ql::kDecMaxSplits + 1];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || S < 1 || S > ql::kDecMaxSplits) return 0;
  if (dev < 64 && known[dev][S].load(std::memory_order_acquire)) return cache[dev][S].load();
  int n = 0;
  if (dec_set_attrs<BN, E8M0, VQ, SF>() == QL_OK) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, 1, 1);
    cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, ql::fp4_decode_kernel<BN, E8M0, VQ, SF>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  if (dev < 64) {
    cache[dev][S].store(n);
    known[dev][S].store(true, std::memory_order_release);
  }
  return n;
}

template <int BN, bool E8M0, bool VQ, int SF = 0>
ql_status launch_dec_bn(const CUtensorMap& tm_x, const ql::DecodeArgs& a, int grid, cudaStream_t s) {
  using Cfg = ql::DecCfg<BN, E8M0, VQ, SF>;
  ql_status st = dec_set_attrs<BN, E8M0, VQ, SF>();
  if (st != QL_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = a.cluster ? a.splits : 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.cluster ? 2 : 1;
  QL_CUDA(cudaLaunchKernelEx(&cfg, ql::fp4_decode_kernel<BN, E8M0, VQ, SF>, tm_x, a));
  return QL_OK;
}

template <bool E8M0, bool VQ, int SF = 0>
ql_status launch_dec(int BN, const CUtensorMap& tm_x, const ql::DecodeArgs& a, int grid, cudaStream_t s) {
  switch (BN) {
    case 16: return launch_dec_bn<16, E8M0, VQ, SF>(tm_x, a, grid, s);
    case 32: return launch_dec_bn<32, E8M0, VQ, SF>(tm_x, a, grid, s);
    case 64: return launch_dec_bn<64, E8M0, VQ, SF>(tm_x, a, grid, s);
  }
  return fail(QL_ERR_UNSUPPORTED, "no decode tile for BN=%d", BN);
}
template <bool E8M0, bool VQ, int SF = 0>
int dec_max_clusters(int BN, int S) {
  switch (BN) {
    case 16: return dec_max_clusters_bn<16, E8M0, VQ, SF>(S);
    case 32: return dec_max_clusters_bn<32, E8M0, VQ, SF>(S);
    default: return dec_max_clusters_bn<64, E8M0, VQ, SF>(S);
  }
}

// Token-tile width: the smallest power of two >= M up to 128.  Past 128 tokens, 256-wide tiles,
// unless the grid has at least one full wave of tiles either way and 160-wide tiles need no more
// waves per unit of operand traffic (each stage streams 128 weight rows plus BN token rows): at
// 2048 tokens x 20 weight tiles, 256 wide gives 160 tiles = 2 waves on 148 SMs, 160 wide gives
// 260 tiles = also 2 waves with 25 % less operand traffic per tile.
int pick_bn(int64_t M, int tiles_n) {
  for (int bn : {16, 32, 64, 128})
    if (M <= bn) return bn;
  const int64_t sms = sm_count();
  auto cost = [&](int bn) -> int64_t {
    const int64_t tiles = tiles_n * cdiv(M, bn);
    return tiles < sms ? -1 : cdiv(tiles, sms) * (128 + bn);
  };
  const int64_t c256 = cost(256), c160 = cost(160);
  return (c256 > 0 && c160 > 0 && c160 < c256) ? 160 : 256;
}

}  // namespace

// ========================================================================= handles
struct ql_linear {
  ql_wformat wfmt;
  int64_t N, K, C;
  int32_t k_tail;
  bool e8m0 = true;            // E8M0-B32 scales (else E4M3-B16 + tensor scales)
  bool vq = false;             // MXCode VQ weight
  int sfmode = 0;              // VQ scales: 0 PreScale atoms, 1 PostScale per QBlock, 2 PreScale+
  int had = 0;                 // online block-32 Hadamard of the activations (MXFP4 layers)
  bool tail_copy = false;      // the quantized activation in the workspace is [Z~, Z~_tail]
  uint8_t* d_scb = nullptr;    // PreScale+: scale codebook [256][8] on the device
  uint8_t* d_codes = nullptr;  // weight blocks [N/128][stages][codes or indices + codebooks, scales]
  size_t weight_bytes = 0;
  float w_ts = 1.f;
  int n_base_stages = 0, n_stages_total = 0;
  // INT4 dense + block-sparse residual
  bool int4 = false;
  int* d_stage_start = nullptr;   // [N/128 + 1]
  int* d_stage_group = nullptr;   // [stages]
  int max_tile_stages = 0;
};

namespace {

// Channels of the quantized activation in the workspace: C, or C + k_tail with the tail copied.
int64_t act_width(const ql_linear* L) { return L->tail_copy ? L->C + L->k_tail : L->C; }

struct FwdPlan {
  int BN, splits, spp, tiles_n, tiles_m;
  int full_tiles;   // FP4 GEMM: tiles [0, full_tiles) unsplit, the rest split `splits` ways
  int sfb_atoms;
  int sf_rows;      // rows per token tile in the tiled activation-scale layout (>= 128)
  size_t sync_off;   // E4M3 grid quantizer: launch counter and per-CTA amax slots
  size_t codes_off, sf_off, scal_off, tick_off, part_off, total;
  int n_tickets;   // split-K tickets (zeroed by the quantizer, re-armed by the GEMM)
  bool decode = false;   // fp4_decode_kernel: M <= 64, one CTA per (weight tile, K range)
  bool fusable = false;  // ... and the forward may quantize x inside it (one launch)
  int fuse_mode = 1;     // 1: cooperatively over the grid; 2: each CTA its own stages
  bool amax_coop = false;   // fuse_mode 2, E4M3: the tensor amax combined over the CTAs
  bool cluster = false;     // the K-splits of a tile form a cluster (fuse_mode 2 or 0)
  size_t dsync_off = 0;  // its launch counter, slots and flags
  size_t xt_off = 0, st_off = 0;   // fused: per-stage B tiles and activation scale sets
};


// Every plan starts with the E4M3-B16 grid quantizer's sync block and the decode kernel's: the
// launch counters there must survive whatever other layers write into a shared workspace.
size_t sync_prefix_bytes() {
  return align_up(align_up(ql::kE4m3SyncBytes, 256) + ql::kDecSyncBytes, 256);
}

FwdPlan plan_forward_int4(const ql_linear* L, int64_t M) {
  FwdPlan p{};
  p.BN = M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128));
  p.tiles_n = static_cast<int>(L->N / 128);
  p.tiles_m = static_cast<int>(cdiv(std::max<int64_t>(M, 1), p.BN));
  const int tiles = p.tiles_n * p.tiles_m;
  const int total = L->max_tile_stages;
  int splits = 1;
  const int target = sm_count();
  if (tiles < target) splits = std::max(1, std::min({total, target / tiles, ql::kInt4MaxClusterSplits}));
  p.spp = static_cast<int>(cdiv(total, splits));
  p.splits = static_cast<int>(cdiv(total, p.spp));
  p.sfb_atoms = p.tiles_m * p.BN;                       // ldt of the transposed scales
  // the sync blocks of the FP4 layers stay reserved, so that layers of different formats can
  // share one workspace without clobbering each other's launch counters
  size_t off = sync_prefix_bytes();
  p.codes_off = off;                                    // int8 activation [M, K]
  off = align_up(off + static_cast<size_t>(M) * L->K, 256);
  p.sf_off = off;                                       // scales [K/128][ldt]
  off = align_up(off + static_cast<size_t>(L->K / 128) * p.sfb_atoms * 4, 256);
  p.scal_off = off;
  p.total = off;
  return p;
}

// Most weight stages one decode CTA keeps resident, per token-tile width and weight format.
template <bool E8M0, bool VQ, int SF = 0>
int dec_max_stages(int BN) {
  switch (BN) {
    case 16: return ql::DecCfg<16, E8M0, VQ, SF>::kMaxStages;
    case 32: return ql::DecCfg<32, E8M0, VQ, SF>::kMaxStages;
    default: return ql::DecCfg<64, E8M0, VQ, SF>::kMaxStages;
  }
}
int dec_max_stages(const ql_linear* L, int BN) {
  if (L->vq && L->sfmode == 1) return dec_max_stages<false, true, 1>(BN);
  if (L->vq && L->sfmode == 2) return dec_max_stages<false, true, 2>(BN);
  if (L->vq) return dec_max_stages<false, true>(BN);
  return L->e8m0 ? dec_max_stages<true, false>(BN) : dec_max_stages<false, false>(BN);
}
int dec_max_clusters(const ql_linear* L, int BN, int S) {
  if (L->vq && L->sfmode == 1) return dec_max_clusters<false, true, 1>(BN, S);
  if (L->vq && L->sfmode == 2) return dec_max_clusters<false, true, 2>(BN, S);
  if (L->vq) return dec_max_clusters<false, true>(BN, S);
  return L->e8m0 ? dec_max_clusters<true, false>(BN, S) : dec_max_clusters<false, false>(BN, S);
}

// Decode-kernel activation quantization: -1 chooses per launch, 1 or 2 forces that mode where
// the launch allows it (ql_decode_fuse_mode).
std::atomic<int> g_decode_fuse_mode{-1};
constexpr int kDecLocalUnits = 8;                // local mode: units per quantizer thread at most
constexpr int64_t kDecLocalAmaxElems = 128 * 1024;   // x elements every CTA may read for the amax
constexpr int64_t kDecClusterAmaxElems = 16 * 1024;  // ... when a cluster exchange is the other way

// Whether a forward of M tokens runs the decode kernel (when it also plans): forced by
// ql_decode_fuse_mode, else by what measured faster on the B200 in chains of CUDA-graph replayed
// layers of 2560 x 9728.  With E4M3-B16 activations (VQ and NVFP4 layers) the separate grid
// quantizer and the general GEMM won from M = 8 up (VQ: 13.9 against 18.6 us at M = 8, 21.3
// against 22.5 at M = 64) and tied at M = 1 (12.6 / 12.5); with MXFP4 activations the decode
// kernel won at M = 1 (9.5 against 10.0) and from M = 64 (14.5 against 16.3) and lost in between.
bool use_decode_kernel(const ql_linear* L, int64_t M) {
  const int forced = g_decode_fuse_mode.load();
  if (forced == 0) return false;
  if (forced > 0) return true;
  if (M == 1) return true;
  return L->e8m0 && !L->vq && M > 32;
}

// Decode launches (M <= 64): the weight tiles split along K so that the grid covers the SMs once;
// each CTA keeps all its stages resident.  Returns false when no such split exists.
bool plan_decode(const ql_linear* L, int64_t M, FwdPlan& p) {
  if (L->int4 || M > 64 || M < 1) return false;
  p.tiles_n = static_cast<int>(cdiv(L->N, 128));
  p.BN = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
  p.tiles_m = 1;
  const int sms = std::min(sm_count(), ql::kDecMaxGrid);
  if (p.tiles_n > sms) return false;
  const int total = L->n_stages_total;
  const int max_stages = dec_max_stages(L, p.BN);   // (VQ: leaves room for one ring tile)
  int splits = std::max(1, std::min({sms / p.tiles_n, total, ql::kDecMaxSplits}));
  p.spp = static_cast<int>(cdiv(total, splits));
  p.splits = static_cast<int>(cdiv(total, p.spp));
  if (p.spp > max_stages) return false;
  // each CTA quantizing its own stages: (stage, row, 32-column) units per quantizer thread
  auto local_ok = [&](int spp) { return cdiv(static_cast<int64_t>(spp) * M * 8, 128) <= kDecLocalUnits; };
  const int forced = g_decode_fuse_mode.load();
  // Preferred: the splits of a tile as one cluster (no grid-wide waits at all), with the largest
  // split count whose clusters the device holds at once.
  p.cluster = false;
  if (forced == -1 || forced == 3) {
    for (int sp = p.splits; sp >= 1; --sp) {
      const int spp = static_cast<int>(cdiv(total, sp));
      const int s2 = static_cast<int>(cdiv(total, spp));
      if (spp > max_stages) break;
      if (s2 != sp) continue;
      if (dec_max_clusters(L, p.BN, s2) >= p.tiles_n) {
        p.spp = spp;
        p.splits = s2;
        p.cluster = true;
        break;
      }
    }
  }
  // fused quantization without a cluster: split z's units (M rows x its 32-column groups) over
  // the split's tiles (cooperative), or each CTA its own stages (local)
  const int64_t upr_max = std::min<int64_t>(static_cast<int64_t>(p.spp) * 8, L->C / 32);
  const bool coop_ok = cdiv(M * upr_max, p.tiles_n) <= 128 * ql::kDecQUnits;
  if (p.cluster) p.fuse_mode = local_ok(p.spp) ? 2 : 0;
  else if (forced == 3) p.fuse_mode = 0;
  else if (forced == 1) p.fuse_mode = coop_ok ? 1 : 0;
  else if (forced == 2) p.fuse_mode = local_ok(p.spp) ? 2 : 0;
  else p.fuse_mode = local_ok(p.spp) ? 2 : (coop_ok ? 1 : 0);
  p.fusable = p.fuse_mode != 0;
  // E4M3: every CTA reads all of x for the tensor amax while x is small, else the grid gathers it
  p.amax_coop = !L->e8m0 && M * L->C > (p.cluster ? kDecClusterAmaxElems : kDecLocalAmaxElems);
  p.full_tiles = 0;
  p.decode = true;
  return true;
}

FwdPlan plan_forward(const ql_linear* L, int64_t M) {
  if (L->int4) return plan_forward_int4(L, M);
  FwdPlan p{};
  if (use_decode_kernel(L, M) && plan_decode(L, M, p)) {
    const int atomK = L->e8m0 ? 128 : 64;
    p.sfb_atoms = static_cast<int>(cdiv(act_width(L), atomK));
    p.sf_rows = 128;
    p.sync_off = 0;   // (the E4M3 grid quantizer of qlinear_quantize_input)
    p.dsync_off = align_up(ql::kE4m3SyncBytes, 256);
    size_t off = sync_prefix_bytes();
    p.codes_off = off;
    off = align_up(off + static_cast<size_t>(M) * (act_width(L) / 2), 256);
    p.sf_off = off;   // one 128-row group of scale atoms (the quantizers write up to 2)
    off = align_up(off + static_cast<size_t>(2) * p.sfb_atoms * 512, 256);
    p.scal_off = off;   // [0] amax bit pattern, [1] tensor scale (E4M3-B16)
    p.tick_off = off + 2 * sizeof(float);
    p.n_tickets = 0;
    off = align_up(p.tick_off, 256);
    p.xt_off = off;     // per K stage: B tile [BN][128 B], then (st) its scale atoms
    off = align_up(off + static_cast<size_t>(L->n_stages_total) * p.BN * 128, 256);
    p.st_off = off;
    off = align_up(off + static_cast<size_t>(L->n_stages_total) * (L->e8m0 ? 2 : 4) * 512, 256);
    p.part_off = off;
    if (p.splits > 1)
      off = align_up(off + static_cast<size_t>(p.tiles_n) * p.splits * p.BN * 128 * 4, 256);
    p.total = off;
    return p;
  }
  p.tiles_n = static_cast<int>(cdiv(L->N, 128));
  p.BN = pick_bn(M, p.tiles_n);
  p.tiles_m = static_cast<int>(cdiv(std::max<int64_t>(M, 1), p.BN));
  const int tiles = p.tiles_n * p.tiles_m;
  const int total = L->n_stages_total;
  // One CTA per SM.  With at least as many tiles as SMs every tile runs unsplit.  With fewer,
  // every tile is split along K so that the grid covers the SMs; the number of ways is bounded
  // by kMaxSplits and by the volume of fp32 partials one tile's last split must add up (about
  // 512 KB).  (Splitting only the tiles left over after the last whole wave was measured too:
  // at 160 prefill tiles on 148 SMs the split tiles' reduction cost more than the idle SMs.)
  const int target = sm_count();
  p.full_tiles = tiles >= target ? tiles : 0;
  const int rest = tiles - p.full_tiles;
  int splits = 1;
  if (rest > 0)
    splits = std::max(1, std::min({total, target / rest, ql::kMaxSplits, std::max(1, 1024 / p.BN)}));
  p.spp = static_cast<int>(cdiv(total, splits));
  p.splits = static_cast<int>(cdiv(total, p.spp));
  const int atomK = L->e8m0 ? 128 : 64;  // K elements covered by one 512-byte scale atom
  p.sfb_atoms = static_cast<int>(cdiv(act_width(L), atomK));
  p.sf_rows = std::max(p.BN, 128);
  // 128-row atom groups of the tiled activation scales: ceil(sf_rows / 128) per token tile
  const int64_t sf_groups = std::max<int64_t>(cdiv(std::max<int64_t>(M, 1), 256) * 2,
                                              static_cast<int64_t>(p.tiles_m) * cdiv(p.sf_rows, 128));
  p.sync_off = 0;
  p.dsync_off = align_up(ql::kE4m3SyncBytes, 256);
  size_t off = sync_prefix_bytes();
  p.codes_off = off;
  off = align_up(off + static_cast<size_t>(M) * (act_width(L) / 2), 256);
  p.sf_off = off;
  off = align_up(off + static_cast<size_t>(sf_groups) * p.sfb_atoms * 512, 256);
  // [0] amax bit pattern and [1] tensor scale of E4M3-B16 activations, then the split-K tickets
  // (one memset or the quantizer clears the whole run before the GEMM).
  p.scal_off = off;
  p.tick_off = off + 2 * sizeof(float);
  p.n_tickets = p.splits > 1 ? rest : 0;
  off = align_up(p.tick_off + static_cast<size_t>(p.n_tickets) * sizeof(int), 256);
  p.part_off = off;
  if (p.splits > 1)
    off = align_up(off + static_cast<size_t>(rest) * p.splits * p.BN * 128 * 4, 256);
  p.total = off;
  return p;
}

// Weight blocks for the FP4 GEMM: for every 128-row tile and every K stage of 256 elements (the
// base stages over [0, C), then the tail stages over [C, C + k_tail)), one block laid out exactly
// as the kernel's stage buffer, so that one bulk copy moves it:
//   FP4: codes as 128 rows x 128 B, 16-byte chunk c of row r stored at chunk c ^ (r % 8) (the
//        128-byte swizzle the MMA reads);
//   VQ:  indices chunk-major, [32-element chunk 8][row 128][8 indices], then the 2 x 4 QBlock
//        codebooks the stage touches (512 B each, row QBlock major);
// then the stage's weight scales as 512-byte atoms of 128 rows x 4 scale columns (row r at
// (r%32)*16 + ((r/32)%4)*4, column j at j%4; the layout tcgen05.cp moves into TMEM).  Rows past N
// and elements past a partial stage are zero.  Returns the block size.
// VQ weights with MXCode PostScale (sfmode 1) or PreScale+ (sfmode 2) scales: the same indices
// and codebooks, then instead of the scale atoms the stage's 8 QBlock scale bytes (2 row QBlocks
// x 4 column QBlocks; 16 bytes with padding) or its 128 x 2 scale indices (row-major).
size_t repack_vq_blocks(const uint8_t* idx, const uint8_t* scales, const uint8_t* lut, int64_t N,
                        int64_t K, int sfmode, std::vector<uint8_t>& out) {
  const int64_t stages = cdiv(K, 256), tiles = cdiv(N, 128);
  const size_t tail = sfmode == 1 ? 16 : 256;
  const size_t blk_bytes = 128 * 64 + 8 * 512 + tail;
  out.assign(static_cast<size_t>(tiles) * stages * blk_bytes, 0);
  for (int64_t t = 0; t < tiles; ++t)
    for (int64_t i = 0; i < stages; ++i) {
      const int64_t kw = i * 256;
      uint8_t* blk = out.data() + (static_cast<size_t>(t) * stages + i) * blk_bytes;
      for (int r = 0; r < 128; ++r) {
        const int64_t n = t * 128 + r;
        if (n >= N) break;
        for (int b = 0; b < 64; ++b) blk[(b >> 3) * 1024 + r * 8 + (b & 7)] = idx[n * (K / 4) + kw / 4 + b];
        if (sfmode == 2)
          for (int g = 0; g < 2; ++g) blk[128 * 64 + 8 * 512 + r * 2 + g] = scales[n * (K / 128) + kw / 128 + g];
      }
      for (int g2 = 0; g2 < 2; ++g2)
        for (int q = 0; q < 4; ++q) {
          const int64_t qr = t * 2 + g2, qc = kw / 64 + q;
          if (qr * 64 < N && qc * 64 < K) {
            std::memcpy(blk + 128 * 64 + g2 * 2048 + q * 512, lut + (static_cast<size_t>(qr) * (K / 64) + qc) * 512, 512);
            if (sfmode == 1) blk[128 * 64 + 8 * 512 + g2 * 4 + q] = scales[qr * (K / 64) + qc];
          }
        }
    }
  return blk_bytes;
}

size_t repack_weight_blocks(const uint8_t* src, const uint8_t* scales, const uint8_t* lut,
                            int64_t N, int64_t K, int64_t C, int64_t k_tail, bool vq, bool e8m0,
                            std::vector<uint8_t>& out) {
  const int64_t nb = cdiv(C, 256), nt = cdiv(k_tail, 256), stages = nb + nt;
  const int64_t tiles = cdiv(N, 128);
  const int row_bytes = vq ? 64 : 128;       // one stage of one row
  const int64_t src_row = vq ? K / 4 : K / 2;
  const int per_byte = vq ? 4 : 2;           // elements per source byte
  const int sfb = e8m0 ? 32 : 16;            // elements per scale
  const int atoms = 256 / (4 * sfb);         // scale atoms per stage
  const size_t code_bytes = static_cast<size_t>(128) * row_bytes;
  const size_t lut_bytes = vq ? 8 * 512 : 0;
  const size_t blk_bytes = code_bytes + lut_bytes + static_cast<size_t>(atoms) * 512;
  out.assign(static_cast<size_t>(tiles) * stages * blk_bytes, 0);
  for (int64_t t = 0; t < tiles; ++t)
    for (int64_t i = 0; i < stages; ++i) {
      int64_t kw, valid;
      if (i < nb) {
        kw = i * 256;
        valid = std::min<int64_t>(256, C - kw);
      } else {
        const int64_t j = (i - nb) * 256;
        kw = C + j;
        valid = std::min<int64_t>(256, k_tail - j);
      }
      uint8_t* blk = out.data() + (static_cast<size_t>(t) * stages + i) * blk_bytes;
      uint8_t* sfa = blk + code_bytes + lut_bytes;
      for (int r = 0; r < 128; ++r) {
        const int64_t n = t * 128 + r;
        if (n >= N) break;
        const uint8_t* srow = src + n * src_row + kw / per_byte;
        const int nbytes = static_cast<int>(valid / per_byte);
        for (int b = 0; b < nbytes; ++b) {
          // VQ: indices chunk-major, [32-element chunk][row][8]; FP4: row-major with the
          // 128-byte swizzle the MMA expects
          const int dst = vq ? ((b >> 3) * 1024 + r * 8 + (b & 7))
                             : (r * row_bytes + ((((b >> 4) ^ (r & 7)) << 4) | (b & 15)));
          blk[dst] = srow[b];
        }
        for (int jl = 0; jl < valid / sfb; ++jl)
          sfa[(jl >> 2) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (jl & 3)] =
              scales[n * (K / sfb) + kw / sfb + jl];
      }
      if (vq)
        for (int g2 = 0; g2 < 2; ++g2)
          for (int q = 0; q < 4; ++q) {
            const int64_t qr = t * 2 + g2, qc = kw / 64 + q;
            if (qr * 64 < N && qc * 64 < K)
              std::memcpy(blk + code_bytes + g2 * 2048 + q * 512,
                          lut + (static_cast<size_t>(qr) * (K / 64) + qc) * 512, 512);
          }
    }
  return blk_bytes;
}

float half_bits_to_float(uint16_t h) {
  const uint32_t sgn = (h & 0x8000u) << 16, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  float f;
  if (e == 0) {
    f = std::ldexp(static_cast<float>(m), -24);
    return sgn ? -f : f;
  }
  const uint32_t u = sgn | (e == 31 ? (0xFFu << 23) : ((e + 112) << 23)) | (m << 13);
  std::memcpy(&f, &u, 4);
  return f;
}

template <int BN>
ql_status launch_int4_bn(const CUtensorMap& tx, const CUtensorMap& ty, const CUtensorMap& ty32,
                         const ql::Int4GemmArgs& a, dim3 grid, cudaStream_t s) {
  using Cfg = ql::Int4Cfg<BN>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    QL_CUDA(cudaFuncSetAttribute(ql::int4_gemm_kernel<BN>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
    attr_done[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = grid.z;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  QL_CUDA(cudaLaunchKernelEx(&cfg, ql::int4_gemm_kernel<BN>, tx, ty, ty32, a));
  return QL_OK;
}

ql_status launch_quant_int4(const void* x, int64_t M, int64_t K, int8_t* q8, uint8_t* q4, float* sc,
                            float* sct, int ldt, cudaStream_t s) {
  const long warps = M * (K / 128);
  if (warps == 0) return QL_OK;
  ql::quant_int4_g128_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<int>(M), static_cast<int>(K), q8, q4, sc,
      sct, ldt);
  QL_CUDA(cudaGetLastError());
  return QL_OK;
}

// k_tail > 0: the outputs are the augmented activation [Z~, Z~_tail] of K + k_tail channels
// (the codes and scales of the last k_tail channels written a second time behind the others).
ql_status launch_quant_mx(const void* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* sp,
                          uint8_t* st, int st_atoms, int* zero_words, int nzero,
                          cudaStream_t s, __nv_bfloat16* deq = nullptr, int st_rows = 128,
                          int had = 0, int64_t k_tail = 0) {
  const long total = static_cast<long>(M) * (K / 32);
  const long threads = std::max<long>(total, nzero);
  if (threads == 0) return QL_OK;
  const int block = 256;
  const long grid = (threads + block - 1) / block;
  const int64_t W = K + k_tail;   // output channels
  ql::quant_mx_e8m0_b32_kernel<<<static_cast<unsigned>(grid), block, 0, s>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<int>(M), static_cast<int>(K),
      static_cast<int>(K), codes, static_cast<int>(W / 2), sp, static_cast<int>(W / 32), st,
      st_atoms, st_rows, zero_words, nzero, deq, had,
      k_tail > 0 ? static_cast<int>(K - k_tail) : -1, static_cast<int>(K));
  QL_CUDA(cudaGetLastError());
  return QL_OK;
}

// Cluster size for the one-launch quantizer: 16 CTAs where the device can co-schedule such a
// cluster, else the portable 8.
int e4m3_cluster_size() {
  static std::atomic<int> size[64] = {};   // 0 until probed; host threads may race to probe
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 8;
  if (size[dev].load(std::memory_order_acquire) == 0) {
    int want = 8;
    if (cudaFuncSetAttribute(ql::quant_e4m3_b16_cluster_kernel,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1, 1);
      cfg.blockDim = dim3(ql::kE4m3ClusterThreads, 1, 1);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, ql::quant_e4m3_b16_cluster_kernel, &cfg) == cudaSuccess &&
          n > 0)
        want = 16;
    }
    cudaGetLastError();
    size[dev].store(want, std::memory_order_release);
  }
  return size[dev].load(std::memory_order_acquire);
}

// Tensors whose 16-element blocks fit the registers of one cluster (kE4m3RegBlocks per thread)
// are quantized in one launch: by one CTA up to 2^14 elements (a single decode token), else by
// one cluster.
constexpr int64_t kE4m3OneCtaMaxElems = int64_t(1) << 14;
bool e4m3_one_launch(int64_t M, int64_t K) {
  const int64_t cap = int64_t(ql::kE4m3RegBlocks) * ql::kE4m3ClusterThreads * 16;   // elements per CTA
  return M * K <= kE4m3OneCtaMaxElems || M * K <= cap * e4m3_cluster_size();
}

// E4M3-B16 activation quantizer.  amax_slot: device word for the reduced amax bit pattern (the
// two-launch path max-reduces into it; it is followed by the tensor-scale word and then
// n_tickets split-K tickets, all cleared here).  ts_out: where ts goes (may be null).
ql_status launch_quant_e4m3(const void* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* sp,
                            uint8_t* st, int st_atoms, unsigned* amax_slot, float* ts_out,
                            cudaStream_t s, int n_tickets = 0, uint32_t* sync = nullptr,
                            int st_rows = 128) {
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  int* tickets = n_tickets > 0 ? reinterpret_cast<int*>(amax_slot + 2) : nullptr;
  // Past one block per thread of a cluster, a grid of small co-resident CTAs when the caller's
  // workspace provides the synchronisation words: it spreads the work over up to one CTA per SM
  // (measured at 64 x 9728: 6.2 us against 9.9 us for the 16-CTA cluster; at 8 x 9728 the
  // cluster's on-chip barrier wins, 5.0 against 5.6 us).
  const int64_t nblocks = M * (K / 16);
  const int64_t grid_cap = std::min<int64_t>(sm_count(), ql::kE4m3GridMaxCtas);
  if (sync != nullptr && M * K > kE4m3OneCtaMaxElems &&
      nblocks > int64_t(e4m3_cluster_size()) * ql::kE4m3ClusterThreads &&
      nblocks <= grid_cap * ql::kE4m3GridThreads * ql::kE4m3RegBlocks) {
    const int g = static_cast<int>(std::min<int64_t>(grid_cap, cdiv(nblocks, ql::kE4m3GridThreads)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g, 1, 1);
    cfg.blockDim = dim3(ql::kE4m3GridThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may start early; waits
    attr[0].val.programmaticStreamSerializationAllowed = 1;            // for x in-kernel
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    QL_CUDA(cudaLaunchKernelEx(&cfg, ql::quant_e4m3_b16_grid_kernel, xb, static_cast<int>(M),
                               static_cast<int>(K), static_cast<int>(K), amax_slot, ts_out, codes,
                               static_cast<int>(K / 2), sp, static_cast<int>(K / 16), st, st_atoms, st_rows,
                               tickets, n_tickets, sync));
    return QL_OK;
  }
  if (e4m3_one_launch(M, K)) {
    const int cs = M * K <= kE4m3OneCtaMaxElems ? 1 : e4m3_cluster_size();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs, 1, 1);
    cfg.blockDim = dim3(ql::kE4m3ClusterThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may start early; waits
    attr[1].val.programmaticStreamSerializationAllowed = 1;            // for x in-kernel
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    QL_CUDA(cudaLaunchKernelEx(&cfg, ql::quant_e4m3_b16_cluster_kernel, xb, static_cast<int>(M),
                               static_cast<int>(K), static_cast<int>(K), amax_slot, ts_out, codes,
                               static_cast<int>(K / 2), sp, static_cast<int>(K / 16), st, st_atoms, st_rows,
                               tickets, n_tickets));
    return QL_OK;
  }
  QL_CUDA(cudaMemsetAsync(amax_slot, 0, sizeof(unsigned) + (n_tickets > 0 ? sizeof(float) + n_tickets * sizeof(int) : 0), s));
  const long n8 = static_cast<long>(M) * K / 8;
  const int block = 256;
  const long want = (n8 + block - 1) / block;
  const int grid_a = static_cast<int>(std::max<long>(1, std::min<long>(want, 4L * sm_count())));
  ql::absmax_bf16_kernel<<<grid_a, block, 0, s>>>(xb, n8, amax_slot);
  QL_CUDA(cudaGetLastError());
  const long total = static_cast<long>(M) * (K / 16);
  ql::quant_e4m3_b16_kernel<<<static_cast<unsigned>((total + block - 1) / block), block, 0, s>>>(
      xb, static_cast<int>(M), static_cast<int>(K), static_cast<int>(K), amax_slot, ts_out, codes,
      static_cast<int>(K / 2), sp, static_cast<int>(K / 16), st, st_atoms, st_rows);
  QL_CUDA(cudaGetLastError());
  return QL_OK;
}

// Tensor-pipe peak probe (measurement only).
template <int KIND, int N>
ql_status launch_peak(int ctas, int iters, cudaStream_t s, double* flops) {
  using Cfg = ql::PeakCfg<KIND, N>;
  auto k = ql::tensor_peak_kernel<KIND, N>;
  QL_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem));
  k<<<ctas, 128, Cfg::kSmem, s>>>(iters);
  QL_CUDA(cudaGetLastError());
  if (flops != nullptr)
    *flops = Cfg::kFlopsPerMma * Cfg::kMmaPerTile * static_cast<double>(iters) * ctas;
  return QL_OK;
}
}  // namespace

extern "C" {

const char* ql_version(void) { return "qlinear-b200 0.1 (sm_100a)"; }
const char* ql_last_error(void) { return g_last_error.c_str(); }

static ql_status create_int4_bsr(const ql_weight_desc* d, cudaStream_t s, ql_linear** out) {
  if (d->codes == nullptr || d->scales == nullptr)
    return fail(QL_ERR_INVALID_ARG, "INT4 layer needs codes and scales");
  if (d->N <= 0 || d->K <= 0 || d->N % 128 != 0 || d->K % 128 != 0 || d->k_tail != 0)
    return fail(QL_ERR_UNSUPPORTED, "INT4 layer needs N %% 128 == 0, K %% 128 == 0, no tail");
  if (d->bsr_nnzb < 0 || (d->bsr_nnzb > 0 && (d->bsr_rowptr == nullptr || d->bsr_col == nullptr ||
                                             d->bsr_codes == nullptr || d->bsr_scales == nullptr)))
    return fail(QL_ERR_INVALID_ARG, "bad block-sparse residual description");
  if (d->bsr_nnzb > 0 && (d->bsr_block_n != 16 || d->bsr_block_k != 128))
    return fail(QL_ERR_UNSUPPORTED, "residual blocks must be 16 x 128");
  const int64_t N = d->N, K = d->K, G = K / 128, tiles = N / 128;
  const uint8_t* codes = static_cast<const uint8_t*>(d->codes);
  const uint16_t* sc = static_cast<const uint16_t*>(d->scales);
  const uint8_t* rcodes = static_cast<const uint8_t*>(d->bsr_codes);
  const uint16_t* rsc = static_cast<const uint16_t*>(d->bsr_scales);
  std::vector<int> start(tiles + 1, 0), group;
  std::vector<uint8_t> blocks;
  blocks.reserve(static_cast<size_t>(tiles) * (G + 8) * ql::kInt4WBlock);
  int max_st = 0;
  for (int64_t t = 0; t < tiles; ++t) {
    start[t] = static_cast<int>(group.size());
    auto add_block = [&](int g) {
      group.push_back(g);
      const size_t at = blocks.size();
      blocks.resize(at + ql::kInt4WBlock, 0);
      return blocks.data() + at;
    };
    for (int g = 0; g < G; ++g) {
      uint8_t* b = add_block(g);
      float* rs = reinterpret_cast<float*>(b + 128 * 64);
      for (int r = 0; r < 128; ++r) {
        const int64_t n = t * 128 + r;
        std::memcpy(b + r * 64, codes + n * (K / 2) + g * 64, 64);
        rs[r] = half_bits_to_float(sc[n * G + g]);
      }
    }
    if (d->bsr_nnzb > 0) {
      std::vector<int> gs;
      for (int nb = static_cast<int>(t * 8); nb < t * 8 + 8; ++nb)
        for (int i = d->bsr_rowptr[nb]; i < d->bsr_rowptr[nb + 1]; ++i) {
          if (i < 0 || i >= d->bsr_nnzb || d->bsr_col[i] < 0 || d->bsr_col[i] >= G)
            return fail(QL_ERR_INVALID_ARG, "residual block index out of range");
          gs.push_back(d->bsr_col[i]);
        }
      std::sort(gs.begin(), gs.end());
      gs.erase(std::unique(gs.begin(), gs.end()), gs.end());
      for (int g : gs) {
        uint8_t* b = add_block(g);
        float* rs = reinterpret_cast<float*>(b + 128 * 64);
        for (int nb = static_cast<int>(t * 8); nb < t * 8 + 8; ++nb)
          for (int i = d->bsr_rowptr[nb]; i < d->bsr_rowptr[nb + 1]; ++i) {
            if (d->bsr_col[i] != g) continue;
            for (int r = 0; r < 16; ++r) {
              const int row = (nb - static_cast<int>(t * 8)) * 16 + r;
              std::memcpy(b + row * 64, rcodes + (static_cast<size_t>(i) * 16 + r) * 64, 64);
              rs[row] = half_bits_to_float(rsc[static_cast<size_t>(i) * 16 + r]);
            }
          }
      }
    }
    max_st = std::max(max_st, static_cast<int>(group.size()) - start[t]);
  }
  start[tiles] = static_cast<int>(group.size());
  auto* L = new ql_linear();
  L->wfmt = d->wfmt;
  L->N = N; L->K = K; L->C = K; L->k_tail = 0;
  L->e8m0 = false; L->int4 = true; L->max_tile_stages = max_st;
  auto cleanup = [&](ql_status st) {
    cudaFree(L->d_codes); cudaFree(L->d_stage_start); cudaFree(L->d_stage_group);
    delete L;
    return st;
  };
  if (cudaMalloc(&L->d_codes, blocks.size()) != cudaSuccess ||
      cudaMalloc(&L->d_stage_start, start.size() * sizeof(int)) != cudaSuccess ||
      cudaMalloc(&L->d_stage_group, group.size() * sizeof(int)) != cudaSuccess)
    return cleanup(fail(QL_ERR_OOM, "cudaMalloc of INT4 weight blocks failed"));
  if (cudaMemcpyAsync(L->d_codes, blocks.data(), blocks.size(), cudaMemcpyHostToDevice, s) ||
      cudaMemcpyAsync(L->d_stage_start, start.data(), start.size() * sizeof(int), cudaMemcpyHostToDevice, s) ||
      cudaMemcpyAsync(L->d_stage_group, group.data(), group.size() * sizeof(int), cudaMemcpyHostToDevice, s) ||
      cudaStreamSynchronize(s))
    return cleanup(fail(QL_ERR_CUDA, "INT4 weight upload failed"));
  *out = L;
  return QL_OK;
}

ql_status qlinear_create(const ql_weight_desc* d, ql_stream_t stream, ql_linear** out) {
  if (d == nullptr || out == nullptr) return fail(QL_ERR_INVALID_ARG, "null descriptor/out");
  *out = nullptr;
  if (d->wfmt == QL_W_INT4_G128_BSR)
    return create_int4_bsr(d, reinterpret_cast<cudaStream_t>(stream), out);
  const bool mx = d->wfmt == QL_W_MXFP4_E8M0_B32;
  const bool nv = d->wfmt == QL_W_NVFP4_E4M3_B16;
  const int sfmode = d->wfmt == QL_W_VQ_POSTSCALE_E4M3_B16 ? 1
                   : d->wfmt == QL_W_VQ_PRESCALE_PLUS_E4M3_B16 ? 2 : 0;
  const bool vq = d->wfmt == QL_W_VQ_PRESCALE_E4M3_B16 || sfmode != 0;
  if (!mx && !nv && !vq)
    return fail(QL_ERR_UNSUPPORTED, "weight format %d not supported by qlinear_create",
                int(d->wfmt));
  if (d->scales == nullptr || (vq ? (d->indices == nullptr || d->codebooks == nullptr)
                                  : d->codes == nullptr))
    return fail(QL_ERR_INVALID_ARG, "codes/indices/codebooks/scales must be non-null host pointers");
  if (d->N <= 0 || d->K <= 0 || d->k_tail < 0 || d->k_tail >= d->K)
    return fail(QL_ERR_INVALID_ARG, "bad sizes N=%lld K=%lld k_tail=%d", (long long)d->N,
                (long long)d->K, d->k_tail);
  if (mx && (d->N % 16 != 0 || d->K % 128 != 0 || d->k_tail % 128 != 0))
    return fail(QL_ERR_UNSUPPORTED, "MXFP4 layer needs N%%16==0, K%%128==0, k_tail%%128==0");
  if (nv && (d->N % 16 != 0 || d->K % 64 != 0 || d->k_tail != 0))
    return fail(QL_ERR_UNSUPPORTED, "E4M3-B16 layer needs N%%16==0, K%%64==0, no tail");
  if (vq && (d->N % 128 != 0 || d->K % 256 != 0 || d->k_tail != 0 || d->qblock_n != 64 ||
             d->qblock_k != 64))
    return fail(QL_ERR_UNSUPPORTED, "VQ layer needs N%%128==0, K%%256==0, 64x64 QBlocks, no tail");
  if ((nv || vq) && !(d->w_tensor_scale > 0.f))
    return fail(QL_ERR_INVALID_ARG, "E4M3-B16 weights need a positive FP32 tensor scale");
  if (sfmode == 2 && (d->scale_codebook == nullptr || d->scale_codebook_entries != 256 ||
                      d->scale_group != 8))
    return fail(QL_ERR_UNSUPPORTED, "PreScale+ needs a scale codebook of 256 entries of 8 scales");
  if (d->had_block != 0 && (d->had_block != 32 || !mx))
    return fail(QL_ERR_UNSUPPORTED, "online Hadamard: block 32 with MXFP4 (E8M0-B32) layers only");
  if (d->tail_copy != 0 && (d->tail_copy != 1 || !mx || d->k_tail == 0))
    return fail(QL_ERR_INVALID_ARG, "tail_copy = 1 needs an MXFP4 layer with k_tail > 0");
  if (d->N > (1 << 24) || d->K > (1 << 24))
    return fail(QL_ERR_UNSUPPORTED, "N/K too large");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto* L = new ql_linear();
  L->wfmt = d->wfmt;
  L->N = d->N;
  L->K = d->K;
  L->k_tail = d->k_tail;
  L->C = d->K - d->k_tail;
  L->e8m0 = mx;
  L->vq = vq;
  L->sfmode = sfmode;
  L->had = d->had_block == 32 ? 1 : 0;
  L->tail_copy = d->tail_copy == 1;
  L->w_ts = mx ? 1.f : d->w_tensor_scale;
  L->n_base_stages = static_cast<int>(cdiv(L->C, 256));
  L->n_stages_total = L->n_base_stages + static_cast<int>(cdiv(L->k_tail, 256));
  std::vector<uint8_t> blocks;
  const size_t blk = sfmode != 0
      ? repack_vq_blocks(static_cast<const uint8_t*>(d->indices), static_cast<const uint8_t*>(d->scales),
                         static_cast<const uint8_t*>(d->codebooks), d->N, d->K, sfmode, blocks)
      : repack_weight_blocks(vq ? static_cast<const uint8_t*>(d->indices)
                                : static_cast<const uint8_t*>(d->codes),
                             static_cast<const uint8_t*>(d->scales),
                             vq ? static_cast<const uint8_t*>(d->codebooks) : nullptr, d->N, d->K,
                             L->C, L->k_tail, vq, mx, blocks);
  const size_t want = sfmode == 1 ? ql::Fp4Cfg<16, false, true, 1>::kWBytes
                    : sfmode == 2 ? ql::Fp4Cfg<16, false, true, 2>::kWBytes
                    : vq ? ql::Fp4Cfg<16, false, true>::kWBytes
                         : (mx ? ql::Fp4Cfg<16, true, false>::kWBytes : ql::Fp4Cfg<16, false, false>::kWBytes);
  if (blk != want) {
    delete L;
    return fail(QL_ERR_UNSUPPORTED, "internal: weight block of %zu bytes, kernel expects %zu", blk, want);
  }
  const size_t code_bytes = blocks.size();
  auto cleanup = [&](ql_status st) {
    if (L->d_codes) cudaFree(L->d_codes);
    if (L->d_scb) cudaFree(L->d_scb);
    delete L;
    return st;
  };
  if (sfmode == 2) {
    if (cudaMalloc(&L->d_scb, 256 * 8) != cudaSuccess)
      return cleanup(fail(QL_ERR_OOM, "cudaMalloc of the scale codebook failed"));
    if (cudaMemcpyAsync(L->d_scb, d->scale_codebook, 256 * 8, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return cleanup(fail(QL_ERR_CUDA, "scale codebook upload failed"));
  }
  if (cudaMalloc(&L->d_codes, code_bytes) != cudaSuccess)
    return cleanup(fail(QL_ERR_OOM, "cudaMalloc of %zu weight bytes failed", code_bytes));
  if (cudaMemcpyAsync(L->d_codes, blocks.data(), code_bytes, cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return cleanup(fail(QL_ERR_CUDA, "weight upload failed"));
  L->weight_bytes = code_bytes;
  *out = L;
  return QL_OK;
}

ql_status qlinear_destroy(ql_linear* L) {
  if (L == nullptr) return QL_OK;
  if (L->d_codes) cudaFree(L->d_codes);
  if (L->d_scb) cudaFree(L->d_scb);
  if (L->d_stage_start) cudaFree(L->d_stage_start);
  if (L->d_stage_group) cudaFree(L->d_stage_group);
  delete L;
  return QL_OK;
}

ql_status qlinear_workspace_bytes(const ql_linear* L, int64_t M, size_t* bytes) {
  if (L == nullptr || bytes == nullptr || M < 0) return fail(QL_ERR_INVALID_ARG, "bad args");
  *bytes = plan_forward(L, M).total;
  return QL_OK;
}

static ql_status check_ws(const ql_linear* L, int64_t M, void* ws, size_t ws_bytes, FwdPlan* p) {
  if (L == nullptr || M < 0) return fail(QL_ERR_INVALID_ARG, "null layer or negative M");
  if (M > (1 << 20)) return fail(QL_ERR_UNSUPPORTED, "M too large");
  *p = plan_forward(L, M);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0 || ws_bytes < p->total)
    return fail(QL_ERR_WORKSPACE, "workspace needs %zu bytes, 256-aligned", p->total);
  return QL_OK;
}

ql_status qlinear_quantize_input(const ql_linear* L, const void* x, int64_t M, void* ws,
                                 size_t ws_bytes, ql_stream_t stream) {
  if (L != nullptr && M == 0) return QL_OK;
  FwdPlan p;
  ql_status st = check_ws(L, M, ws, ws_bytes, &p);
  if (st != QL_OK) return st;
  if (x == nullptr) return fail(QL_ERR_INVALID_ARG, "null x");
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0)
    return fail(QL_ERR_INVALID_ARG, "x must be 16-byte aligned");
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  if (L->int4)
    return launch_quant_int4(x, M, L->K, reinterpret_cast<int8_t*>(w8 + p.codes_off), nullptr,
                             nullptr, reinterpret_cast<float*>(w8 + p.sf_off), p.sfb_atoms,
                             reinterpret_cast<cudaStream_t>(stream));
  if (!L->e8m0) {
    unsigned* scal = reinterpret_cast<unsigned*>(w8 + p.scal_off);
    return launch_quant_e4m3(x, M, L->C, w8 + p.codes_off, nullptr, w8 + p.sf_off, p.sfb_atoms,
                             scal, reinterpret_cast<float*>(scal + 1),
                             reinterpret_cast<cudaStream_t>(stream), p.n_tickets,
                             reinterpret_cast<uint32_t*>(w8 + p.sync_off), p.sf_rows);
  }
  return launch_quant_mx(x, M, L->C, w8 + p.codes_off, nullptr, w8 + p.sf_off, p.sfb_atoms,
                         reinterpret_cast<int*>(w8 + p.tick_off), p.n_tickets,
                         reinterpret_cast<cudaStream_t>(stream), nullptr, p.sf_rows, L->had,
                         L->tail_copy ? L->k_tail : 0);
}

// The decode kernel: x != null quantizes x inside it (qlinear_forward), else the workspace holds
// the quantized activations (qlinear_quantize_input, then qlinear_gemm).
static ql_status launch_decode(const ql_linear* L, int64_t M, const FwdPlan& p, const void* x,
                               void* y, float* y32, uint8_t* w8, ql_stream_t stream) {
  ql::DecodeArgs a{};
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(L->N);
  a.C = static_cast<int>(L->C);
  a.k_tail = L->k_tail;
  a.n_base_stages = L->n_base_stages;
  a.n_stages_total = L->n_stages_total;
  a.spp = p.spp;
  a.splits = p.splits;
  a.fuse = x != nullptr ? p.fuse_mode : 0;
  a.amax_coop = p.amax_coop ? 1 : 0;
  a.cluster = p.cluster ? 1 : 0;
  a.act_aug = L->tail_copy ? 1 : 0;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.xq = w8 + p.codes_off;
  a.sfb = w8 + p.sf_off;
  a.xt = w8 + p.xt_off;
  a.st = w8 + p.st_off;
  a.ts_x = reinterpret_cast<float*>(w8 + p.scal_off) + 1;
  a.alpha = L->w_ts;
  a.wt = L->d_codes;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.y32 = y32;
  a.ldy = static_cast<int>(L->N);
  a.partials = reinterpret_cast<float*>(w8 + p.part_off);
  a.sync = w8 + p.dsync_off;
  a.scb = L->d_scb;
  a.had = L->had;
  const int grid = p.tiles_n * p.splits;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap tm_x;   // the plain-layout activation codes (read only when x is quantized already)
  std::memset(&tm_x, 0, sizeof(tm_x));
  if (x == nullptr) {
    ql_status st = make_tmap_u8(&tm_x, w8 + p.codes_off, act_width(L) / 2, M, act_width(L) / 2, 128, p.BN);
    if (st != QL_OK) return st;
  }
  if (L->vq && L->sfmode == 1) return launch_dec<false, true, 1>(p.BN, tm_x, a, grid, cs);
  if (L->vq && L->sfmode == 2) return launch_dec<false, true, 2>(p.BN, tm_x, a, grid, cs);
  if (L->vq) return launch_dec<false, true>(p.BN, tm_x, a, grid, cs);
  if (!L->e8m0) return launch_dec<false, false>(p.BN, tm_x, a, grid, cs);
  return launch_dec<true, false>(p.BN, tm_x, a, grid, cs);
}

ql_status qlinear_gemm(const ql_linear* L, int64_t M, void* y, float* y32, void* ws,
                       size_t ws_bytes, ql_stream_t stream) {
  if (L != nullptr && M == 0) return QL_OK;
  FwdPlan p;
  ql_status st = check_ws(L, M, ws, ws_bytes, &p);
  if (st != QL_OK) return st;
  if (y == nullptr) return fail(QL_ERR_INVALID_ARG, "null y");
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  if (L->int4) {
    if ((reinterpret_cast<uintptr_t>(y) & 15) != 0 || (y32 && (reinterpret_cast<uintptr_t>(y32) & 15)))
      return fail(QL_ERR_INVALID_ARG, "y / y_f32 must be 16-byte aligned");
    CUtensorMap tx, ty, ty32;
    st = make_tmap_u8(&tx, w8 + p.codes_off, L->K, M, L->K, 128, p.BN);
    if (st == QL_OK) st = make_tmap_out(&ty, y, false, L->N, M, L->N, p.BN);
    if (st == QL_OK) st = make_tmap_out(&ty32, y32 ? static_cast<const void*>(y32) : y, y32 != nullptr,
                                        L->N, M, L->N, p.BN);
    if (st != QL_OK) return st;
    ql::Int4GemmArgs a{};
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(L->N);
    a.wblocks = L->d_codes;
    a.stage_start = L->d_stage_start;
    a.stage_group = L->d_stage_group;
    a.sx_t = reinterpret_cast<const float*>(w8 + p.sf_off);
    a.ldt = p.sfb_atoms;
    a.stages_per_split = p.spp;
    a.y = static_cast<__nv_bfloat16*>(y);
    a.y32 = y32;
    dim3 grid(p.tiles_n, p.tiles_m, p.splits);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    switch (p.BN) {
      case 16: return launch_int4_bn<16>(tx, ty, ty32, a, grid, cs);
      case 32: return launch_int4_bn<32>(tx, ty, ty32, a, grid, cs);
      case 64: return launch_int4_bn<64>(tx, ty, ty32, a, grid, cs);
      default: return launch_int4_bn<128>(tx, ty, ty32, a, grid, cs);
    }
  }
  if (p.decode) return launch_decode(L, M, p, nullptr, y, y32, w8, stream);
  CUtensorMap tm_x;
  st = make_tmap_u8(&tm_x, w8 + p.codes_off, act_width(L) / 2, M, act_width(L) / 2, 128, p.BN);
  if (st != QL_OK) return st;
  ql::Fp4GemmArgs a{};
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(L->N);
  a.C = static_cast<int>(L->C);
  a.k_tail = L->k_tail;
  a.n_base_stages = L->n_base_stages;
  a.n_stages_total = L->n_stages_total;
  a.stages_per_split = p.spp;
  a.sfb = w8 + p.sf_off;
  a.sfb_atoms = p.sfb_atoms;
  a.alpha_dev = L->e8m0 ? nullptr : reinterpret_cast<const float*>(w8 + p.scal_off) + 1;
  a.alpha = L->w_ts;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.y32 = y32;
  a.ldy = static_cast<int>(L->N);
  a.wt = L->d_codes;
  a.partials = reinterpret_cast<float*>(w8 + p.part_off);
  a.tickets = reinterpret_cast<int*>(w8 + p.tick_off);
  a.xq = w8 + p.codes_off;
  a.tiles_n = p.tiles_n;
  a.full_tiles = p.full_tiles;
  a.splits = p.splits;
  dim3 grid(p.full_tiles + (p.tiles_n * p.tiles_m - p.full_tiles) * p.splits, 1, 1);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if ((reinterpret_cast<uintptr_t>(y) & 15) != 0 || (y32 && (reinterpret_cast<uintptr_t>(y32) & 15)) ||
      (L->N * 2) % 16 != 0)
    return fail(QL_ERR_INVALID_ARG, "y / y_f32 must be 16-byte aligned");
  CUtensorMap tm_y, tm_y32;
  st = make_tmap_out(&tm_y, y, false, L->N, M, L->N, p.BN);
  if (st == QL_OK) st = make_tmap_out(&tm_y32, y32 ? static_cast<const void*>(y32) : y, y32 != nullptr,
                                      L->N, M, L->N, p.BN);
  if (st != QL_OK) return st;
  a.scb = L->d_scb;
  a.act_aug = L->tail_copy ? 1 : 0;
  if (L->vq && L->sfmode == 1) return launch_fp4<false, true, 1>(p.BN, tm_x, tm_y, tm_y32, a, grid, cs);
  if (L->vq && L->sfmode == 2) return launch_fp4<false, true, 2>(p.BN, tm_x, tm_y, tm_y32, a, grid, cs);
  if (L->vq) return launch_fp4<false, true>(p.BN, tm_x, tm_y, tm_y32, a, grid, cs);
  if (!L->e8m0) return launch_fp4<false, false>(p.BN, tm_x, tm_y, tm_y32, a, grid, cs);
  return launch_fp4<true, false>(p.BN, tm_x, tm_y, tm_y32, a, grid, cs);
}

ql_status qlinear_forward(const ql_linear* L, const void* x, int64_t M, void* y, float* y32,
                          void* ws, size_t ws_bytes, ql_stream_t stream) {
  if (L == nullptr || M < 0) return fail(QL_ERR_INVALID_ARG, "null layer or negative M");
  if (M == 0) return QL_OK;
  if (x == nullptr || y == nullptr) return fail(QL_ERR_INVALID_ARG, "null x/y");
  {
    FwdPlan p;
    ql_status st = check_ws(L, M, ws, ws_bytes, &p);
    if (st != QL_OK) return st;
    if (p.decode && p.fusable) {   // one launch: the activations are quantized inside the GEMM
      if ((reinterpret_cast<uintptr_t>(x) & 15) != 0)
        return fail(QL_ERR_INVALID_ARG, "x must be 16-byte aligned");
      return launch_decode(L, M, p, x, y, y32, static_cast<uint8_t*>(ws), stream);
    }
  }
  ql_status st = qlinear_quantize_input(L, x, M, ws, ws_bytes, stream);
  if (st != QL_OK) return st;
  return qlinear_gemm(L, M, y, y32, ws, ws_bytes, stream);
}

ql_status quantize_act(ql_aformat fmt, const void* x, int64_t M, int64_t K, void* codes,
                       void* scales, float* tensor_scale, ql_stream_t stream) {
  (void)tensor_scale;
  if (M < 0 || K < 0) return fail(QL_ERR_INVALID_ARG, "negative size");
  if (M == 0 || K == 0) return QL_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr)
    return fail(QL_ERR_INVALID_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0 || (reinterpret_cast<uintptr_t>(codes) & 15) != 0)
    return fail(QL_ERR_INVALID_ARG, "x and codes must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (fmt) {
    case QL_A_MXFP4_E8M0_B32:
      if (K % 32 != 0) return fail(QL_ERR_UNSUPPORTED, "MXFP4 needs K %% 32 == 0");
      return launch_quant_mx(x, M, K, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                             nullptr, 0, nullptr, 0, s);
    case QL_A_FP4_E4M3_B16_TS: {
      if (K % 16 != 0) return fail(QL_ERR_UNSUPPORTED, "E4M3-B16 needs K %% 16 == 0");
      if (tensor_scale == nullptr)
        return fail(QL_ERR_INVALID_ARG, "E4M3-B16 needs a device tensor_scale pointer");
      unsigned* slot = reinterpret_cast<unsigned*>(tensor_scale);
      if (e4m3_one_launch(M, K))   // one launch writes ts directly
        return launch_quant_e4m3(x, M, K, static_cast<uint8_t*>(codes),
                                 static_cast<uint8_t*>(scales), nullptr, 0, nullptr, tensor_scale, s);
      ql_status st = launch_quant_e4m3(x, M, K, static_cast<uint8_t*>(codes),
                                       static_cast<uint8_t*>(scales), nullptr, 0, slot, nullptr, s);
      if (st != QL_OK) return st;
      ql::amax_to_tensor_scale_kernel<<<1, 1, 0, s>>>(slot);
      QL_CUDA(cudaGetLastError());
      return QL_OK;
    }
    case QL_A_INT4_TOK_G128:
      if (K % 128 != 0) return fail(QL_ERR_UNSUPPORTED, "INT4 activations need K %% 128 == 0");
      return launch_quant_int4(x, M, K, nullptr, static_cast<uint8_t*>(codes),
                               static_cast<float*>(scales), nullptr, 0, s);
    default:
      return fail(QL_ERR_UNSUPPORTED, "activation format %d not supported", int(fmt));
  }
}

ql_status ql_tensor_peak(int32_t kind, int32_t n, int32_t iters, int32_t ctas,
                         double* flops_per_launch, ql_stream_t stream) {
  if (iters <= 0 || ctas <= 0 || ctas > 4096) return fail(QL_ERR_INVALID_ARG, "iters/ctas");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int key = kind * 1000 + n;
  switch (key) {
    case 0 * 1000 + 128: return launch_peak<0, 128>(ctas, iters, s, flops_per_launch);
    case 0 * 1000 + 256: return launch_peak<0, 256>(ctas, iters, s, flops_per_launch);
    case 1 * 1000 + 128: return launch_peak<1, 128>(ctas, iters, s, flops_per_launch);
    case 1 * 1000 + 256: return launch_peak<1, 256>(ctas, iters, s, flops_per_launch);
    case 2 * 1000 + 128: return launch_peak<2, 128>(ctas, iters, s, flops_per_launch);
    case 2 * 1000 + 256: return launch_peak<2, 256>(ctas, iters, s, flops_per_launch);
    case 3 * 1000 + 128: return launch_peak<3, 128>(ctas, iters, s, flops_per_launch);
    case 3 * 1000 + 256: return launch_peak<3, 256>(ctas, iters, s, flops_per_launch);
    default: return fail(QL_ERR_UNSUPPORTED, "tensor peak kind %d with N %d", int(kind), int(n));
  }
}

ql_status ql_debug_inject(int32_t withhold_cta, uint64_t wait_limit_ns) {
  if (withhold_cta < -1) return fail(QL_ERR_INVALID_ARG, "withhold_cta must be >= -1");
  const unsigned long long lim = wait_limit_ns == 0 ? 2000000000ull : wait_limit_ns;
  const int cta = withhold_cta;
  QL_CUDA(cudaDeviceSynchronize());   // no launch in flight sees a half-changed setting
  QL_CUDA(cudaMemcpyToSymbol(ql::g_wait_limit_ns, &lim, sizeof(lim)));
  QL_CUDA(cudaMemcpyToSymbol(ql::g_debug_withhold_cta, &cta, sizeof(cta)));
  return QL_OK;
}

ql_status ql_decode_fuse_mode(int32_t mode) {
  if (mode < -1 || mode > 3) return fail(QL_ERR_INVALID_ARG, "mode must be -1, 0, 1, 2 or 3");
  g_decode_fuse_mode.store(mode);
  return QL_OK;
}

ql_status quantize_act_augmented(ql_aformat fmt, const void* x, int64_t M, int64_t C,
                                 int32_t k_tail, void* codes, void* scales, ql_stream_t stream) {
  if (M < 0 || C < 0 || k_tail < 0) return fail(QL_ERR_INVALID_ARG, "negative size");
  if (fmt != QL_A_MXFP4_E8M0_B32)
    return fail(QL_ERR_UNSUPPORTED, "the augmented activation is MXFP4 (E8M0-B32) only");
  if (C % 32 != 0 || k_tail % 32 != 0 || k_tail > C)
    return fail(QL_ERR_UNSUPPORTED, "needs C %% 32 == 0, k_tail %% 32 == 0, k_tail <= C");
  if (M == 0 || C == 0) return QL_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return fail(QL_ERR_INVALID_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0 || (reinterpret_cast<uintptr_t>(codes) & 15) != 0)
    return fail(QL_ERR_INVALID_ARG, "x and codes must be 16-byte aligned");
  return launch_quant_mx(x, M, C, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                         nullptr, 0, nullptr, 0, reinterpret_cast<cudaStream_t>(stream), nullptr,
                         128, 0, k_tail);
}

ql_status quantize_act_hadamard(ql_aformat fmt, int32_t had_block, const void* x, int64_t M,
                                int64_t K, void* codes, void* scales, ql_stream_t stream) {
  if (M < 0 || K < 0) return fail(QL_ERR_INVALID_ARG, "negative size");
  if (fmt != QL_A_MXFP4_E8M0_B32 || had_block != 32)
    return fail(QL_ERR_UNSUPPORTED, "online Hadamard: block 32 before MXFP4 (E8M0-B32) only");
  if (K % 32 != 0) return fail(QL_ERR_UNSUPPORTED, "MXFP4 needs K %% 32 == 0");
  if (M == 0 || K == 0) return QL_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr) return fail(QL_ERR_INVALID_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0 || (reinterpret_cast<uintptr_t>(codes) & 15) != 0)
    return fail(QL_ERR_INVALID_ARG, "x and codes must be 16-byte aligned");
  return launch_quant_mx(x, M, K, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                         nullptr, 0, nullptr, 0, reinterpret_cast<cudaStream_t>(stream), nullptr,
                         128, 1);
}

ql_status ql_check(ql_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  QL_CUDA(cudaStreamSynchronize(s));
  int err = 0, site = 0, zero = 0;
  QL_CUDA(cudaMemcpyFromSymbol(&err, ql::g_dev_error, sizeof(int)));
  QL_CUDA(cudaMemcpyFromSymbol(&site, ql::g_dev_error_site, sizeof(int)));
  if (err != 0) {
    QL_CUDA(cudaMemcpyToSymbol(ql::g_dev_error, &zero, sizeof(int)));
    return fail(QL_ERR_TIMEOUT, "device wait expired (code %d, site %d)", err, site);
  }
  return QL_OK;
}

}  // extern "C"

// ========================================================================= MoE
struct ql_moe {
  int E, k, H, I;
  uint8_t* d_idx_gu = nullptr;        // [E*2I, H/2] 4-bit indices, kernel row order
  uint8_t* d_idx_d = nullptr;         // [E*H, I/2]
  __nv_bfloat16* d_cent_gu = nullptr; // [E*2I][16]
  __nv_bfloat16* d_cent_d = nullptr;  // [E*H][16]
  CUtensorMap tm_idx_gu, tm_idx_d;
  bool capture_h32 = false;
  int had_x = 0, had_h = 0;           // online block-32 Hadamard of x (gate/up) and of h (down)
};

namespace {

constexpr int kMoeBN = 128;   // tokens per work item (N of the MMA; 256 measured slower)

struct MoePlan {
  size_t counts, offsets, entries, ids, gates, x_codes, x_scales, x_dq, xs, h_codes, h_scales,
      h_dq, h32, yslot, total;
};

MoePlan plan_moe(const ql_moe* m, int64_t T) {
  MoePlan p{};
  const size_t P = static_cast<size_t>(T) * m->k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + std::max<size_t>(bytes, 1), 256);
    return o;
  };
  p.counts = take(sizeof(int) * m->E);
  p.offsets = take(sizeof(int) * (m->E + 1));
  p.entries = take(sizeof(int) * P);
  p.ids = take(sizeof(int) * P);
  p.gates = take(sizeof(float) * P);
  p.x_codes = take(static_cast<size_t>(T) * m->H / 2);
  p.x_scales = take(static_cast<size_t>(T) * m->H / 32);
  p.x_dq = take(static_cast<size_t>(T) * m->H * 2);
  p.xs = take(P * m->H * 2);   // x rows per routed entry, expert-sorted
  p.h_codes = take(P * m->I / 2);
  p.h_scales = take(P * m->I / 32);
  p.h_dq = take(P * m->I * 2);
  p.h32 = take(m->capture_h32 ? P * m->I * 4 : 0);
  p.yslot = take(P * m->H * 4);
  p.total = off;
  return p;
}

template <int BN, bool GATEUP>
ql_status launch_moe_gemm(const CUtensorMap& ti, const CUtensorMap& tb, const ql::MoeGemmArgs& a,
                          int max_items, cudaStream_t s) {
  using Cfg = ql::MoeCfg<BN>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    QL_CUDA(cudaFuncSetAttribute(ql::moe_gemm_kernel<BN, GATEUP>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
    attr_done[dev] = true;
  }
  // persistent: one CTA per SM (the item count is only known on the device)
  const int grid = std::max(1, std::min(max_items, sm_count()));
  ql::moe_gemm_kernel<BN, GATEUP><<<grid, Cfg::kThreads, Cfg::kSmemBytes, s>>>(ti, tb, a);
  QL_CUDA(cudaGetLastError());
  return QL_OK;
}

}  // namespace

extern "C" {

ql_status moe_create(const ql_weight_desc* gu, const ql_weight_desc* dn, int32_t E, int32_t top_k,
                     ql_stream_t stream, ql_moe** out) {
  if (gu == nullptr || dn == nullptr || out == nullptr) return fail(QL_ERR_INVALID_ARG, "null args");
  *out = nullptr;
  if (gu->wfmt != QL_W_CLUSTER4_ROW16_BF16 || dn->wfmt != QL_W_CLUSTER4_ROW16_BF16)
    return fail(QL_ERR_UNSUPPORTED, "MoE experts must use QL_W_CLUSTER4_ROW16_BF16");
  if (E <= 0 || E > 256 || top_k <= 0 || top_k > 16 || top_k > E)
    return fail(QL_ERR_UNSUPPORTED, "need 0 < top_k <= 16, top_k <= E <= 256");
  if (gu->codes == nullptr || gu->codebooks == nullptr || dn->codes == nullptr ||
      dn->codebooks == nullptr)
    return fail(QL_ERR_INVALID_ARG, "codes and codebooks must be non-null host pointers");
  if (gu->N % E != 0 || dn->N % E != 0) return fail(QL_ERR_INVALID_ARG, "N must be E * rows");
  const int64_t two_i = gu->N / E, H = gu->K, I = dn->K;
  if (dn->N / E != H || two_i != 2 * I)
    return fail(QL_ERR_INVALID_ARG, "gate/up must be [E*2I, H] and down [E*H, I]");
  if (I % 64 != 0 || H % 128 != 0 || H % 64 != 0 || I < 64)
    return fail(QL_ERR_UNSUPPORTED, "MoE needs I %% 64 == 0 and H %% 128 == 0");
  if ((gu->had_block != 0 && gu->had_block != 32) || (dn->had_block != 0 && dn->had_block != 32))
    return fail(QL_ERR_UNSUPPORTED, "online Hadamard: block 32 only");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto* m = new ql_moe();
  m->E = E; m->k = top_k; m->H = static_cast<int>(H); m->I = static_cast<int>(I);
  m->had_x = gu->had_block == 32 ? 1 : 0;
  m->had_h = dn->had_block == 32 ? 1 : 0;
  // gate/up rows in kernel order: per expert, per 128-row tile: 64 gate rows then the 64 up
  // rows with the same intermediate index, so SwiGLU pairs sit in one accumulator tile.
  const size_t rgu = static_cast<size_t>(E) * two_i;
  std::vector<uint8_t> idx_gu(rgu * (H / 2));
  std::vector<uint16_t> cent_gu(rgu * 16);
  const uint8_t* src_idx = static_cast<const uint8_t*>(gu->codes);
  const uint16_t* src_c = static_cast<const uint16_t*>(gu->codebooks);
  for (int64_t e = 0; e < E; ++e)
    for (int64_t r = 0; r < two_i; ++r) {
      const int64_t tile = r / 128, w = r % 128;
      const int64_t srow = (w < 64) ? tile * 64 + w : I + tile * 64 + (w - 64);
      const size_t d = e * two_i + r, sr = e * two_i + srow;
      std::memcpy(&idx_gu[d * (H / 2)], src_idx + sr * (H / 2), H / 2);
      std::memcpy(&cent_gu[d * 16], src_c + sr * 16, 32);
    }
  const size_t rd = static_cast<size_t>(E) * H;
  auto cleanup = [&](ql_status st) {
    cudaFree(m->d_idx_gu); cudaFree(m->d_idx_d); cudaFree(m->d_cent_gu); cudaFree(m->d_cent_d);
    delete m;
    return st;
  };
  if (cudaMalloc(&m->d_idx_gu, idx_gu.size()) != cudaSuccess ||
      cudaMalloc(&m->d_idx_d, rd * (I / 2)) != cudaSuccess ||
      cudaMalloc(&m->d_cent_gu, cent_gu.size() * 2) != cudaSuccess ||
      cudaMalloc(&m->d_cent_d, rd * 32) != cudaSuccess)
    return cleanup(fail(QL_ERR_OOM, "cudaMalloc of MoE weights failed"));
  if (cudaMemcpyAsync(m->d_idx_gu, idx_gu.data(), idx_gu.size(), cudaMemcpyHostToDevice, s) ||
      cudaMemcpyAsync(m->d_idx_d, dn->codes, rd * (I / 2), cudaMemcpyHostToDevice, s) ||
      cudaMemcpyAsync(m->d_cent_gu, cent_gu.data(), cent_gu.size() * 2, cudaMemcpyHostToDevice, s) ||
      cudaMemcpyAsync(m->d_cent_d, dn->codebooks, rd * 32, cudaMemcpyHostToDevice, s) ||
      cudaStreamSynchronize(s))
    return cleanup(fail(QL_ERR_CUDA, "MoE weight upload failed"));
  ql_status st = make_tmap_u8(&m->tm_idx_gu, m->d_idx_gu, H / 2, rgu, H / 2, 32, 128, false);
  if (st == QL_OK) st = make_tmap_u8(&m->tm_idx_d, m->d_idx_d, I / 2, rd, I / 2, 32, 128, false);
  if (st != QL_OK) return cleanup(st);
  *out = m;
  return QL_OK;
}

ql_status moe_destroy(ql_moe* m) {
  if (m == nullptr) return QL_OK;
  cudaFree(m->d_idx_gu); cudaFree(m->d_idx_d); cudaFree(m->d_cent_gu); cudaFree(m->d_cent_d);
  delete m;
  return QL_OK;
}

ql_status moe_capture_intermediate(ql_moe* m, int32_t enable) {
  if (m == nullptr) return fail(QL_ERR_INVALID_ARG, "null moe");
  m->capture_h32 = enable != 0;
  return QL_OK;
}

ql_status moe_workspace_bytes(const ql_moe* m, int64_t T, size_t* bytes) {
  if (m == nullptr || bytes == nullptr || T < 0) return fail(QL_ERR_INVALID_ARG, "bad args");
  *bytes = plan_moe(m, T).total;
  return QL_OK;
}

ql_status moe_workspace_layout(const ql_moe* m, int64_t T, ql_moe_ws_layout* out) {
  if (m == nullptr || out == nullptr || T < 0) return fail(QL_ERR_INVALID_ARG, "bad args");
  const MoePlan p = plan_moe(m, T);
  out->counts = p.counts; out->offsets = p.offsets; out->entries = p.entries; out->ids = p.ids;
  out->gates = p.gates; out->x_codes = p.x_codes; out->x_scales = p.x_scales; out->x_dq = p.x_dq;
  out->h_codes = p.h_codes; out->h_scales = p.h_scales; out->h_dq = p.h_dq;
  out->h32 = m->capture_h32 ? p.h32 : SIZE_MAX; out->yslot = p.yslot; out->total = p.total;
  return QL_OK;
}

ql_status moe_grouped_forward(const ql_moe* m, const void* x, int64_t T, const float* logits,
                              void* y, float* y32, int32_t* ids_out, float* gates_out, void* ws,
                              size_t ws_bytes, ql_stream_t stream) {
  if (m == nullptr || T < 0) return fail(QL_ERR_INVALID_ARG, "null moe or negative T");
  if (T == 0) return QL_OK;
  if (x == nullptr || logits == nullptr || y == nullptr)
    return fail(QL_ERR_INVALID_ARG, "null x/logits/y");
  if (T > (1 << 20)) return fail(QL_ERR_UNSUPPORTED, "T too large");
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0 || (reinterpret_cast<uintptr_t>(y) & 15) != 0)
    return fail(QL_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
  const MoePlan p = plan_moe(m, T);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0 || ws_bytes < p.total)
    return fail(QL_ERR_WORKSPACE, "workspace needs %zu bytes, 256-aligned", p.total);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  int* counts = reinterpret_cast<int*>(w8 + p.counts);
  int* offsets = reinterpret_cast<int*>(w8 + p.offsets);
  int* entries = reinterpret_cast<int*>(w8 + p.entries);
  int* ids = reinterpret_cast<int*>(w8 + p.ids);
  float* gates = reinterpret_cast<float*>(w8 + p.gates);
  const int total = static_cast<int>(T * m->k);
  QL_CUDA(cudaMemsetAsync(counts, 0, sizeof(int) * m->E, s));
  ql::moe_topk_kernel<<<static_cast<unsigned>((T * 32 + 255) / 256), 256, 0, s>>>(
      logits, static_cast<int>(T), m->E, m->k, ids, gates, counts);
  QL_CUDA(cudaGetLastError());
  ql::moe_scatter_kernel<<<m->E, ql::kScatterThreads, 0, s>>>(ids, total, m->E, counts, offsets, entries);
  QL_CUDA(cudaGetLastError());
  __nv_bfloat16* x_dq = reinterpret_cast<__nv_bfloat16*>(w8 + p.x_dq);
  ql_status st = launch_quant_mx(x, T, m->H, w8 + p.x_codes, w8 + p.x_scales, nullptr, 0, nullptr,
                                 0, s, x_dq, 128, m->had_x);
  if (st != QL_OK) return st;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(w8 + p.xs);
  {
    const long n16 = static_cast<long>(total) * (m->H / 8);
    ql::moe_gather_kernel<<<static_cast<unsigned>((n16 + 255) / 256), 256, 0, s>>>(
        x_dq, entries, total, m->H, m->k, xs);
    QL_CUDA(cudaGetLastError());
  }
  CUtensorMap tm_x, tm_h;
  __nv_bfloat16* h_dq = reinterpret_cast<__nv_bfloat16*>(w8 + p.h_dq);
  st = make_tmap_bf16(&tm_x, xs, m->H, total, kMoeBN);
  if (st == QL_OK) st = make_tmap_bf16(&tm_h, h_dq, m->I, total, kMoeBN);
  if (st != QL_OK) return st;
  ql::MoeGemmArgs a{};
  a.E = m->E; a.k = m->k; a.counts = counts; a.offsets = offsets; a.entries = entries;
  a.gates = gates; a.I = m->I; a.H = m->H;
  a.h_codes = w8 + p.h_codes; a.h_scales = w8 + p.h_scales; a.h_dq = h_dq;
  a.h32 = m->capture_h32 ? reinterpret_cast<float*>(w8 + p.h32) : nullptr;
  a.yslot = reinterpret_cast<float*>(w8 + p.yslot);
  a.had = m->had_h;
  const int max_mtiles = m->E + (total + kMoeBN - 1) / kMoeBN;   // >= sum_e ceil(count_e / BN)
  a.rows_per_expert = 2 * m->I; a.kdim = m->H; a.n_tiles = 2 * m->I / 128; a.cent = m->d_cent_gu;
  st = launch_moe_gemm<kMoeBN, true>(m->tm_idx_gu, tm_x, a, a.n_tiles * max_mtiles, s);
  if (st != QL_OK) return st;
  a.rows_per_expert = m->H; a.kdim = m->I; a.n_tiles = m->H / 128; a.cent = m->d_cent_d;
  st = launch_moe_gemm<kMoeBN, false>(m->tm_idx_d, tm_h, a, a.n_tiles * max_mtiles, s);
  if (st != QL_OK) return st;
  const long n4 = T * m->H / 4;
  ql::moe_combine_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, s>>>(
      a.yslot, static_cast<int>(T), m->H, m->k, static_cast<__nv_bfloat16*>(y), y32);
  QL_CUDA(cudaGetLastError());
  if (ids_out != nullptr)
    QL_CUDA(cudaMemcpyAsync(ids_out, ids, sizeof(int) * total, cudaMemcpyDeviceToDevice, s));
  if (gates_out != nullptr)
    QL_CUDA(cudaMemcpyAsync(gates_out, gates, sizeof(float) * total, cudaMemcpyDeviceToDevice, s));
  return QL_OK;
}

}  // extern "C"

// Sets the message that ql_last_error() returns on this thread and passes the status through
// (used by entry points that live in other source files of the library).
ql_status ql_set_error(ql_status status, const char* message) {
  return fail(status, "%s", message);
}
