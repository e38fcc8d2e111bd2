// qlora.cu -- host side of the library: argument validation, workspace layout, TMA tensor maps,
// kernel launches and the extern "C" entry points declared in include/qlora.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "qlora.h"
#include "qlora_debug.cuh"
#include "qlora_fused.cuh"
#include "qlora_lora.cuh"
#include "qlora_stream.cuh"
#include "qlora_short.cuh"
#include "qlora_w4a8.cuh"
#include <algorithm>
#include <utility>
#include "qlora_quant.cuh"
#include "qlora_loftq.cuh"

namespace qlora {
namespace {

// ------------------------------------------------------------------------------------ helpers
// Workspace header, cleared by qlora_workspace_init: [0] device status word, [1] pair-kernel
// ticket, bytes [64, 192) lora_down's arrival counters of a multi-cluster split, bytes
// [256, 8192) the short-batch kernels' arrival counters, 4 per tile (each launch leaves all
// counters at zero).
constexpr size_t kHeaderBytes = 8192;
constexpr size_t kCounterOffset = 256;
constexpr size_t kDownCountOffset = 64;
constexpr int kDownCounters = 32;
// The no-alloc forward's scratch holds only the status word and the ticket in its header.
constexpr size_t kNoAllocHeaderBytes = 256;
constexpr int kMaxClusterSplits = 8;        // split-K CTAs of one LoRA tile (one portable cluster)
// CTAs of a lora_down launch that feeds the pair kernel: the pair kernel starts beside it on the
// other SMs and waits for its output only at the end of its first tile
constexpr int kDownCtasBesidePair = 32;
// The same for the short-batch streaming kernel, which up to 64 rows also leaves that many SMs to
// lora_down (its ranges are equal, so a late CTA would delay the whole launch)
constexpr int kDownCtasBesideStream = 16;
// U = dY B ahead of the short-batch dX kernel: the whole contraction (N deep) on one 128-row
// tile, which one cluster of 8 CTAs takes ~0.35 us per 64-deep step to stream; up to this many
// CTAs (clusters of 8) split it, their sums added through the workspace.  The dX kernel's CTAs
// that find no free SM start when these end, a few microseconds later.
constexpr int kDownWideCtas = 64;
constexpr int kMaxDownClusters = kDownWideCtas / kMaxClusterSplits;
static_assert(kMaxClusterSplits <= kDownCounters, "one tile's counters fit the header");
constexpr int kMaxDevices = 64;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int rank_pad(int r) { return (r + 15) / 16 * 16; }
bool rank_ok(int r) { return r == 8 || r == 16 || r == 32 || r == 64; }

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

int num_sms() {
  static std::atomic<int> cache[kMaxDevices] = {};   // threads may race to fill it: same value
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  int v = cache[d].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || v <= 0) v = 148;
    cache[d].store(v, std::memory_order_relaxed);
  }
  return v;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D row-major tensor [outer, inner] (inner contiguous, row pitch in bytes), box {bi, bo}.
bool tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
             uint64_t outer, uint64_t pitch_bytes, uint32_t bi, uint32_t bo, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {bi, bo};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle swizzle_for_bytes(uint32_t b) {
  return b == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                  : (b == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

template <typename K>
bool set_smem(K kernel, size_t bytes) {
  // Both attributes persist per kernel and device, so each (kernel, device) is set once, to the
  // largest size asked for so far; later launches that ask no more make no driver call.  Every
  // kernel of the library asks for the largest shared-memory carveout, so that consecutive
  // launches never make the SMs switch their L1 / shared-memory split.
  struct Entry {
    const void* fn;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const void* fn = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lk(mu);
  Entry* hit = nullptr;
  for (Entry& e : done)
    if (e.fn == fn && e.dev == dev) hit = &e;
  if (hit && hit->bytes >= bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess ||
      cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return false;
  if (hit) hit->bytes = bytes;
  else done.push_back(Entry{fn, dev, bytes});
  return true;
}

// Launch with programmatic stream serialization: the kernel may begin while the previous kernel of
// the stream runs; it waits for it (griddepcontrol.wait) after its own prologue.
template <typename P>
cudaError_t launch_pdl(void (*kernel)(P), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       const P& params) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, params);
}

// As launch_pdl, with the grid cut into thread-block clusters of `cluster` CTAs along x (1: no
// clusters).
template <typename P>
cudaError_t launch_pdl_cluster(void (*kernel)(P), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t st, const P& params, unsigned cluster) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, params);
}

qlora_status_t check_weight(const qlora_weight_t* W) {
  if (!W) return QLORA_ERR_INVALID_ARG;
  if (W->fmt < QLORA_FMT_NF4 || W->fmt > QLORA_FMT_NF4_DQ) return QLORA_ERR_INVALID_ARG;
  if (W->N < 16 || W->N % 16 != 0 || W->K < 64 || W->K % 64 != 0) return QLORA_ERR_INVALID_ARG;
  if (W->N > (int64_t(1) << 30) || W->K > (int64_t(1) << 30)) return QLORA_ERR_INVALID_ARG;
  if (!W->codes || !W->scales || !aligned16(W->codes) || !aligned16(W->scales))
    return QLORA_ERR_INVALID_ARG;
  if (W->fmt == QLORA_FMT_NVFP4 &&
      (!W->tensor_scale || (reinterpret_cast<uintptr_t>(W->tensor_scale) & 3u)))
    return QLORA_ERR_INVALID_ARG;
  if (W->fmt == QLORA_FMT_NF4_DQ &&
      (!W->scales2 || (reinterpret_cast<uintptr_t>(W->scales2) & 3u)))
    return QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}

bool ptr_ok(const void* p) { return p && aligned16(p); }

// ------------------------------------------------------------------------------- workspace
// E = number of experts (1 for a single layer); M = all rows.
// Reduction plan of the dA/dB kernel: per expert, tiles of 128 rows of N (dB) and of K (dA); each
// expert's rows split into S ranges of whole 64-row chunks (the ranges are resolved on the device
// from the offsets).
struct WgradPlan {
  int tiles0, tiles1, S;
};

WgradPlan wgrad_plan(int64_t N, int64_t K, int64_t M, int E, int sms) {
  WgradPlan p{};
  p.tiles0 = int((N + 127) / 128);
  p.tiles1 = int((K + 127) / 128);
  const int64_t tiles = int64_t(E) * (p.tiles0 + p.tiles1);
  int S = int(sms / tiles);                                  // at most one wave of long splits
  S = S < 1 ? 1 : (S > kMaxClusterSplits ? kMaxClusterSplits : S);
  const int64_t chunks = (M + 63) / 64;                      // of one expert holding every row
  if (S > chunks) S = chunks > 0 ? int(chunks) : 1;
  p.S = S;
  return p;
}

// Split plan of the lora_down kernel: 128-row tiles (at most ceil(M/128) + E - 1 over all
// experts), the contraction (Kc) split into S ranges of whole 64-deep steps, >= 2 steps each.
// wide > 0 (one layer of one tile, S = 8): C = min(wide / 8, steps / 16) clusters of S CTAs
// split it S * C ways (trailing splits may be empty), C * 128 * rpad fp32 sums in the workspace.
struct DownPlan {
  int tiles, S, C, sps, num_k;
};

DownPlan down_plan(int64_t M, int64_t Kc, int E, int ctas, int wide) {
  DownPlan p{};
  p.tiles = int((M + 127) / 128) + (E > 1 ? E - 1 : 0);
  p.num_k = int((Kc + 63) / 64);
  int S = p.tiles > 0 ? ctas / p.tiles : 1;                  // at most `ctas` CTAs of long splits
  S = S < 1 ? 1 : (S > kMaxClusterSplits ? kMaxClusterSplits : S);
  const int max_s = p.num_k / 2 > 0 ? p.num_k / 2 : 1;
  if (S > max_s) S = max_s;
  p.C = 1;
  if (wide > 0 && E == 1 && p.tiles == 1 && S == kMaxClusterSplits) {
    int C = wide / S;
    const int max_c = p.num_k / (2 * S);
    C = C > max_c ? max_c : C;
    C = C > kMaxDownClusters ? kMaxDownClusters : C;
    p.C = C < 1 ? 1 : C;
  }
  if (p.C > 1) {
    p.sps = (p.num_k + S * p.C - 1) / (S * p.C);
    p.S = S;
  } else {
    p.sps = (p.num_k + S - 1) / S;
    p.S = (p.num_k + p.sps - 1) / p.sps;
  }
  return p;
}

// Workspace bytes of lora_down's cluster sums for a multi-cluster U of rank r (and any M).
size_t down_sum_bytes(int r) {
  return size_t(kMaxDownClusters) * 128 * size_t(rank_pad(r)) * 4;
}

// Short batches (M <= 256 rows, one weight) use the weight-streaming kernels: the flat space of
// (256-column output tile, 64-deep step) iterations, plus one LoRA step per tile, cut into equal
// contiguous ranges, one per CTA.
struct StreamPlan {
  int tiles, nk, iters, grid, segments;
  long long lcm;
  size_t partial_bytes;
};

bool use_stream(int64_t M, int E) { return E == 1 && M > 0 && M <= stream::kMaxRows; }

StreamPlan stream_plan(int64_t N, int64_t K, int64_t M, bool dx, int sms) {
  StreamPlan p{};
  // Up to 64 rows the launch is short next to lora_down: leave it its SMs.  Above, the decode
  // work per SM is larger than lora_down's duration is worth.
  if (M <= 64 && sms > 4 * kDownCtasBesideStream) sms -= kDownCtasBesideStream;
  p.tiles = int(((dx ? K : N) + stream::BN - 1) / stream::BN);
  p.nk = int(((dx ? N : K) + stream::BK - 1) / stream::BK);
  const int64_t total = int64_t(p.tiles) * (p.nk + 1);
  int64_t L = (total + sms - 1) / sms;
  if (L < 2) L = 2;
  p.iters = int(L);
  p.grid = int((total + L - 1) / L);
  const int64_t nk1 = p.nk + 1;
  int64_t a = L, b = nk1;
  while (b) { const int64_t t = a % b; a = b; b = t; }
  p.lcm = L / a * nk1;
  p.segments = int(p.grid + p.tiles - (total + p.lcm - 1) / p.lcm);
  p.partial_bytes = size_t(p.segments) * size_t(M) * stream::BN * 4;
  return p;
}

// The streaming path is taken when the batch is short and the workspace's partial region (all
// of the workspace from its start) holds its fp32 partials; otherwise the tiled kernels run.
bool stream_fits(const qlora_weight_t* W, int64_t M, int E, bool dx, size_t region) {
  // NF4 with a double-quantised absmax runs the tiled kernels at every batch size
  return W->fmt != QLORA_FMT_NF4_DQ && use_stream(M, E) &&
         stream_plan(W->N, W->K, M, dx, num_sms()).partial_bytes <= region;
}

// Batches of at most 64 rows (one weight, NF4 / MXFP4 / NVFP4) use the short-batch kernels: the
// flat space of (output tile, 64-deep step) iterations plus one LoRA step per tile, cut into equal
// contiguous ranges, one per CTA; pieces of split tiles go to fp32 partials [tiles][pieces][M][tile
// columns].  The SMs the launch leaves free run lora_down beside it.
struct ShortPlan {
  int tiles, nk, iters, grid, max_pieces, tile_cols;
  size_t partial_bytes;
};

ShortPlan short_plan(int64_t N, int64_t K, int64_t M, bool dx, int sms) {
  ShortPlan p{};
  if (sms > 4 * kDownCtasBesideStream) sms -= kDownCtasBesideStream;
  p.tile_cols = dx ? shortk::D_TILE : shortk::F_TILE;
  p.tiles = int(((dx ? K : N) + p.tile_cols - 1) / p.tile_cols);
  // contraction iterations: 256 weight columns (forward) or 128 weight rows (dX)
  p.nk = int(dx ? (N + 127) / 128 : (K + 255) / 256);
  const int64_t nk1 = p.nk + 1;
  const int64_t total = int64_t(p.tiles) * nk1;
  int64_t L = (total + sms - 1) / sms;
  if (L < 2) L = 2;
  p.iters = int(L);
  p.grid = int((total + L - 1) / L);
  int mp = 1;
  for (int64_t t = 0; t < p.tiles; ++t) {
    const int64_t first = t * nk1 / L, last = (t * nk1 + nk1 - 1) / L;
    if (last - first + 1 > mp) mp = int(last - first + 1);
  }
  p.max_pieces = mp;
  p.partial_bytes = size_t(p.tiles) * size_t(mp) * size_t(M) * size_t(p.tile_cols) * 4;
  return p;
}

bool use_short(const qlora_weight_t* W, int64_t M, int E) {
  return E == 1 && M > 0 && M <= shortk::kMaxRows && W->fmt != QLORA_FMT_NF4_DQ;
}

bool short_fits(const qlora_weight_t* W, int64_t M, int E, bool dx, size_t region) {
  if (!use_short(W, M, E)) return false;
  const ShortPlan sp = short_plan(W->N, W->K, M, dx, num_sms());
  return sp.tiles <= shortk::kMaxTiles && sp.partial_bytes <= region;
}

struct WsLayout {
  size_t zs, t, u, dsum, partial, partial_bytes, total;
};

WsLayout ws_layout(int64_t N, int64_t K, int64_t M, int r, bool bwd, int E, int sms) {
  WsLayout L{};
  size_t off = kHeaderBytes;
  const size_t mr = align_up(size_t(M > 0 ? M : 0) * size_t(r) * 2, 256);
  L.zs = off; off += mr;
  L.t = off; off += mr;
  L.u = off; off += bwd ? mr : 0;
  L.dsum = off; off += (bwd && E == 1) ? down_sum_bytes(r) : 0;   // independent of M
  L.partial = off;
  // fp32 partials of the short-batch weight-streaming kernels
  size_t pb = 0;
  if (E == 1 && M > 0 && M <= shortk::kMaxRows) {
    const size_t sf = short_plan(N, K, M, false, sms).partial_bytes;
    pb = sf > pb ? sf : pb;
    if (bwd) {
      const size_t sd = short_plan(N, K, M, true, sms).partial_bytes;
      pb = sd > pb ? sd : pb;
    }
  }
  if (use_stream(M, E)) {
    const size_t sf = stream_plan(N, K, M, false, sms).partial_bytes;
    pb = sf > pb ? sf : pb;
    if (bwd) {
      const size_t sd = stream_plan(N, K, M, true, sms).partial_bytes;
      pb = sd > pb ? sd : pb;
    }
  }
  L.partial_bytes = align_up(pb, 256);
  off += L.partial_bytes;
  L.total = off;
  return L;
}

int* ws_status(void* ws) { return reinterpret_cast<int*>(ws); }

// ---------------------------------------------------------------------------------- profiling
enum Kind : int {
  kKindFusedFwd = 0, kKindFusedDx, kKindDownT, kKindDownU, kKindWgrad,
  kKindGFusedFwd, kKindGFusedDx, kKindGDownT, kKindGDownU, kKindGWgrad,
  kKindStreamFwd, kKindStreamDx, kKindStreamReduce, kKindShortFwd, kKindShortDx,
  kKindW4a8Quant, kKindW4a8Gemm, kNumKinds
};
const char* const kKindNames[kNumKinds] = {
    "fused_fwd", "fused_dx", "lora_down_T", "lora_down_U", "lora_wgrad",
    "grouped_fused_fwd", "grouped_fused_dx", "grouped_lora_down_T", "grouped_lora_down_U",
    "grouped_lora_wgrad", "stream_fwd", "stream_dx", "stream_reduce", "short_fwd", "short_dx",
    "w4a8_quant", "w4a8_gemm"};
constexpr int kMaxProfiled = 65536;

std::atomic<int64_t> g_launches{0};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<cudaEvent_t> g_ev;          // 2 per record
std::vector<int> g_rec_kind;

// Brackets one kernel launch: counts it, and records start/end events while profiling is on.
struct LaunchScope {
  int slot = -1;
  cudaStream_t st;
  LaunchScope(int kind, cudaStream_t s) : st(s) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (!g_prof_on) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    const int n = int(g_rec_kind.size());
    if (!g_prof_on || 2 * (n + 1) > int(g_ev.size())) return;
    slot = n;
    g_rec_kind.push_back(kind);
    cudaEventRecord(g_ev[2 * n], st);
  }
  ~LaunchScope() {
    if (slot >= 0) cudaEventRecord(g_ev[2 * slot + 1], st);
  }
};

// ---------------------------------------------------------------------------------- launches
// 3-D row-major tensor [d2, d1, d0] (d0 contiguous), box {b0, b1, 1}.
bool tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
             uint32_t b1, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Z = Act . R for every expert's rows: R is A [E, r, Kc] (r_mn false, T = X A^T) or
// B [E, Kc, r] (r_mn true, U = dY B).  offsets == nullptr: one expert of M rows.  beside_pair:
// max_ctas > 0: the next launch of the stream (pair or streaming kernel) runs beside this one,
// which then uses at most that many CTAs.  wide > 0: a one-tile layer may use up to `wide` CTAs
// in several clusters, whose sums go to `sums` (down_sum_bytes) and whose arrival counters are
// the workspace header's (`header`).
qlora_status_t launch_lora_down(bool r_mn, const void* act, int64_t M, int64_t Kc, const void* R,
                                int r, float s, const float* ts, void* z, void* zs, int* status,
                                const int32_t* offsets, int E, bool grouped, int max_ctas,
                                cudaStream_t st, float zs_mul = 1.0f, int wide = 0,
                                void* sums = nullptr, void* header = nullptr) {
  DownParams p{};
  const int rpad = rank_pad(r);
  const DownPlan dp = down_plan(M, Kc, E, max_ctas > 0 ? max_ctas : num_sms(),
                                sums && header ? wide : 0);
  if (!tmap_2d(&p.tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, uint64_t(Kc), uint64_t(M),
               uint64_t(Kc) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  const bool okm = !r_mn
      ? tmap_3d(&p.tm_r, R, uint64_t(Kc), uint64_t(r), uint64_t(E), 64, uint32_t(rpad),
                CU_TENSOR_MAP_SWIZZLE_128B)
      : tmap_3d(&p.tm_r, R, uint64_t(r), uint64_t(Kc), uint64_t(E), uint32_t(rpad), 64,
                swizzle_for_bytes(uint32_t(rpad) * 2));
  if (!okm) return QLORA_ERR_CUDA;
  p.tensor_scale = ts;
  p.z = static_cast<__nv_bfloat16*>(z);
  p.zs = static_cast<__nv_bfloat16*>(zs);
  p.status = status;
  p.offsets = offsets;
  p.M = int(M);
  p.r = r;
  p.rpad = rpad;
  p.num_k = dp.num_k;
  p.S = dp.S;
  p.C = dp.C;
  p.steps_per_split = dp.sps;
  p.E = E;
  p.s = s;
  p.zs_mul = zs_mul;
  if (dp.C > 1) {
    p.cpart = static_cast<float*>(sums);
    p.ccount = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(header) + kDownCountOffset);
  }
  const dim3 grid(unsigned(dp.tiles * dp.S * dp.C));
  const size_t smem = lora::smem_bytes(E);
  LaunchScope scope(grouped ? (r_mn ? kKindGDownU : kKindGDownT) : (r_mn ? kKindDownU : kKindDownT), st);
  if (r_mn) {
    if (!set_smem(qlora_lora_down_kernel<true>, smem)) return QLORA_ERR_CUDA;
    if (launch_pdl_cluster(qlora_lora_down_kernel<true>, grid, dim3(lora::kThreads), smem, st, p,
                           unsigned(dp.S)) != cudaSuccess)
      return QLORA_ERR_CUDA;
  } else {
    if (!set_smem(qlora_lora_down_kernel<false>, smem)) return QLORA_ERR_CUDA;
    if (launch_pdl_cluster(qlora_lora_down_kernel<false>, grid, dim3(lora::kThreads), smem, st, p,
                           unsigned(dp.S)) != cudaSuccess)
      return QLORA_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

template <int FMT, bool DX>
qlora_status_t launch_fused_t(const FusedParams& p, int grid, bool grouped, cudaStream_t st) {
  const size_t smem = fused::smem_bytes(p.E);
  if (!set_smem(qlora_fused_gemm_kernel<FMT, DX>, smem)) return QLORA_ERR_CUDA;
  LaunchScope scope(grouped ? (DX ? kKindGFusedDx : kKindGFusedFwd) : (DX ? kKindFusedDx : kKindFusedFwd), st);
  if (launch_pdl(qlora_fused_gemm_kernel<FMT, DX>, dim3(grid), dim3(fused::kThreads), smem, st, p) !=
      cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// W: one weight (E = 1) or E stacked weights; lora_up: B [E, N, r] (forward) or A [E, r, K] (dX).
qlora_status_t launch_fused(const qlora_weight_t* W, bool dx, const void* act, const void* zs,
                            const void* lora_up, void* out, int64_t M, int r, int* status,
                            const int32_t* offsets, int E, bool grouped, cudaStream_t st) {
  FusedParams p{};
  const int64_t N = W->N, K = W->K;
  const int64_t Kc = dx ? N : K;
  if (!tmap_2d(&p.tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, uint64_t(Kc), uint64_t(M),
               uint64_t(Kc) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  if (!dx) {
    if (!tmap_2d(&p.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, uint64_t(K / 2),
                 uint64_t(N) * uint64_t(E), uint64_t(K / 2), 32, 128, CU_TENSOR_MAP_SWIZZLE_32B))
      return QLORA_ERR_CUDA;
  } else {
    if (!tmap_2d(&p.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, uint64_t(K / 2),
                 uint64_t(N) * uint64_t(E), uint64_t(K / 2), 64, 64, CU_TENSOR_MAP_SWIZZLE_64B))
      return QLORA_ERR_CUDA;
  }
  if (!tmap_2d(&p.tm_zs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, zs, uint64_t(r), uint64_t(M),
               uint64_t(r) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  p.scales = W->scales;
  p.scales2 = W->fmt == QLORA_FMT_NF4_DQ ? W->scales2 : nullptr;
  p.tensor_scale = W->fmt == QLORA_FMT_NVFP4 ? W->tensor_scale : nullptr;
  p.lora_up = static_cast<const __nv_bfloat16*>(lora_up);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.offsets = offsets;
  p.status = status;
  p.ticket = reinterpret_cast<unsigned*>(status + 1);
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.r = r;
  p.E = E;
  p.num_n = int(((dx ? K : N) + fused::BN - 1) / fused::BN);
  p.num_k = int((Kc + fused::BK - 1) / fused::BK);
  // one CTA pair per pair tile, at most one pair per two SMs (persistent beyond that); the tile
  // count of a grouped launch is known only on the device: at most ceil(M/256) + E - 1 row tiles
  int64_t tiles = ((M + fused::BM - 1) / fused::BM + (E > 1 ? E - 1 : 0)) * p.num_n;
  int64_t pairs = tiles < num_sms() / 2 ? tiles : num_sms() / 2;
  // One layer whose last wave of tiles would leave most pairs idle: split that wave's 512-row
  // tiles in two 256-row tiles each, scheduled last, so the wave takes about half as long.
  p.tail_split = 0;
  if (!grouped && E == 1 && pairs > 0) {
    const int64_t rem = tiles % pairs;
    if (rem > 0 && 2 * rem <= pairs && tiles > pairs) p.tail_split = int(rem);
  }
  tiles += p.tail_split;
  pairs = tiles < num_sms() / 2 ? tiles : num_sms() / 2;
  const int grid = int(2 * (pairs > 0 ? pairs : 1));
  switch (W->fmt * 2 + (dx ? 1 : 0)) {
    case 0: return launch_fused_t<kFmtNF4, false>(p, grid, grouped, st);
    case 1: return launch_fused_t<kFmtNF4, true>(p, grid, grouped, st);
    case 2: return launch_fused_t<kFmtMXFP4, false>(p, grid, grouped, st);
    case 3: return launch_fused_t<kFmtMXFP4, true>(p, grid, grouped, st);
    case 4: return launch_fused_t<kFmtNVFP4, false>(p, grid, grouped, st);
    case 5: return launch_fused_t<kFmtNVFP4, true>(p, grid, grouped, st);
    case 6: return launch_fused_t<kFmtNF4DQ, false>(p, grid, grouped, st);
    default: return launch_fused_t<kFmtNF4DQ, true>(p, grid, grouped, st);
  }
}

template <int FMT, bool DX, int MT>
qlora_status_t launch_stream_t(const StreamParams& p, int grid, cudaStream_t st) {
  const size_t smem = stream::smem_bytes(p.xrows);
  if (!set_smem(qlora_stream_gemm_kernel<FMT, DX, MT>, smem)) return QLORA_ERR_CUDA;
  LaunchScope scope(DX ? kKindStreamDx : kKindStreamFwd, st);
  if (launch_pdl(qlora_stream_gemm_kernel<FMT, DX, MT>, dim3(grid), dim3(stream::kThreads), smem, st,
                 p) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// Short-batch path of the fused GEMM (same operands and result as launch_fused with one expert):
// the streaming kernel writes fp32 partials into `partial`, the reduce kernel writes `out`.
qlora_status_t launch_stream(const qlora_weight_t* W, bool dx, const void* act, const void* zs,
                             const void* lora_up, void* out, int64_t M, int r, int* status,
                             float* partial, size_t partial_bytes, cudaStream_t st) {
  const int64_t N = W->N, K = W->K;
  const int64_t Kc = dx ? N : K;
  const StreamPlan sp = stream_plan(N, K, M, dx, num_sms());
  if (sp.partial_bytes > partial_bytes) return QLORA_ERR_WORKSPACE;
  StreamParams p{};
  p.xrows = int((M + 15) / 16 * 16);
  const int mt = p.xrows <= 128 ? 1 : 2;
  if (!tmap_2d(&p.tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, uint64_t(Kc), uint64_t(M),
               uint64_t(Kc) * 2, 64, uint32_t(p.xrows), CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  const bool okc = !dx
      ? tmap_2d(&p.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, uint64_t(K / 2), uint64_t(N),
                uint64_t(K / 2), 32, 128, CU_TENSOR_MAP_SWIZZLE_32B)
      : tmap_2d(&p.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, uint64_t(K / 2), uint64_t(N),
                uint64_t(K / 2), 64, 64, CU_TENSOR_MAP_SWIZZLE_64B);
  if (!okc) return QLORA_ERR_CUDA;
  if (!tmap_2d(&p.tm_zs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, zs, uint64_t(r), uint64_t(M),
               uint64_t(r) * 2, 64, uint32_t(p.xrows), CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  p.scales = W->scales;
  p.lora_up = static_cast<const __nv_bfloat16*>(lora_up);
  p.partial = partial;
  p.status = status;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.r = r;
  p.num_k = sp.nk;
  p.num_tiles = sp.tiles;
  p.iters = sp.iters;
  p.lcm = sp.lcm;
  p.segments = sp.segments;
  qlora_status_t rc;
  switch ((W->fmt * 2 + (dx ? 1 : 0)) * 2 + (mt - 1)) {
    case 0: rc = launch_stream_t<kFmtNF4, false, 1>(p, sp.grid, st); break;
    case 1: rc = launch_stream_t<kFmtNF4, false, 2>(p, sp.grid, st); break;
    case 2: rc = launch_stream_t<kFmtNF4, true, 1>(p, sp.grid, st); break;
    case 3: rc = launch_stream_t<kFmtNF4, true, 2>(p, sp.grid, st); break;
    case 4: rc = launch_stream_t<kFmtMXFP4, false, 1>(p, sp.grid, st); break;
    case 5: rc = launch_stream_t<kFmtMXFP4, false, 2>(p, sp.grid, st); break;
    case 6: rc = launch_stream_t<kFmtMXFP4, true, 1>(p, sp.grid, st); break;
    case 7: rc = launch_stream_t<kFmtMXFP4, true, 2>(p, sp.grid, st); break;
    case 8: rc = launch_stream_t<kFmtNVFP4, false, 1>(p, sp.grid, st); break;
    case 9: rc = launch_stream_t<kFmtNVFP4, false, 2>(p, sp.grid, st); break;
    case 10: rc = launch_stream_t<kFmtNVFP4, true, 1>(p, sp.grid, st); break;
    default: rc = launch_stream_t<kFmtNVFP4, true, 2>(p, sp.grid, st); break;
  }
  if (rc != QLORA_OK) return rc;
  StreamReduceParams rp{};
  rp.partial = partial;
  rp.tensor_scale = W->fmt == QLORA_FMT_NVFP4 ? W->tensor_scale : nullptr;
  rp.out = static_cast<__nv_bfloat16*>(out);
  rp.M = int(M);
  rp.ncols = int(dx ? K : N);
  rp.num_tiles = sp.tiles;
  rp.nk1 = sp.nk + 1;
  rp.iters = sp.iters;
  {
    const long long total = (long long)sp.tiles * (sp.nk + 1);
    rp.lcm = int(sp.lcm < total + 1 ? sp.lcm : total + 1);
  }
  rp.segments = sp.segments;
  const int64_t threads = M * int64_t(sp.tiles) * (stream::BN / 4);
  if (!set_smem(qlora_stream_reduce_kernel, 0)) return QLORA_ERR_CUDA;
  LaunchScope scope(kKindStreamReduce, st);
  if (launch_pdl(qlora_stream_reduce_kernel, dim3(unsigned((threads + 255) / 256)), dim3(256), 0, st,
                 rp) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// NVFP4 runs the short-batch kernels with its elements decoded times 2^-8: Zs carries the same
// factor and the kernels' epilogue multiplies by 2^8 times the tensor scale.
constexpr float kShortNvZsMul = 1.0f / 256.0f;
float short_zs_mul(const qlora_weight_t* W) { return W->fmt == QLORA_FMT_NVFP4 ? kShortNvZsMul : 1.0f; }

template <int FMT, bool DX>
qlora_status_t launch_short_t(const ShortParams& p, int grid, cudaStream_t st) {
  const size_t smem = DX ? shortk::dx_smem_bytes() : shortk::fwd_smem_bytes(p.xrows);
  auto kern = DX ? qlora_short_dx_kernel<FMT> : qlora_short_fwd_kernel<FMT>;
  if (!set_smem(kern, smem)) return QLORA_ERR_CUDA;
  LaunchScope scope(DX ? kKindShortDx : kKindShortFwd, st);
  if (launch_pdl(kern, dim3(grid), dim3(shortk::kThreads), smem, st, p) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// Short-batch path of the fused GEMM (same operands and result as launch_fused with one expert,
// Zs written by lora_down with zs_mul = short_zs_mul(W)).
qlora_status_t launch_short(const qlora_weight_t* W, bool dx, const void* act, const void* zs,
                            const void* lora_up, void* out, int64_t M, int r, void* ws,
                            float* partial, size_t partial_bytes, cudaStream_t st) {
  const int64_t N = W->N, K = W->K;
  const int64_t Kc = dx ? N : K;
  const ShortPlan sp = short_plan(N, K, M, dx, num_sms());
  if (sp.partial_bytes > partial_bytes || sp.tiles > shortk::kMaxTiles) return QLORA_ERR_WORKSPACE;
  ShortParams p{};
  p.xrows = int((M + 15) / 16 * 16);
  if (!tmap_2d(&p.tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, uint64_t(Kc), uint64_t(M),
               uint64_t(Kc) * 2, 64, uint32_t(p.xrows), CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  if (!tmap_2d(&p.tm_zs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, zs, uint64_t(r), uint64_t(M),
               uint64_t(r) * 2, 64, uint32_t(p.xrows), CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  if (!tmap_2d(&p.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, uint64_t(K / 2), uint64_t(N),
               uint64_t(K / 2), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  p.codes = static_cast<const uint8_t*>(W->codes);
  p.scales = W->scales;
  p.tensor_scale = W->fmt == QLORA_FMT_NVFP4 ? W->tensor_scale : nullptr;
  p.lora_up = static_cast<const __nv_bfloat16*>(lora_up);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.partial = partial;
  p.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) + kCounterOffset);
  p.status = ws_status(ws);
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.r = r;
  p.rpad = rank_pad(r);
  p.num_k = sp.nk;
  p.num_tiles = sp.tiles;
  p.iters = sp.iters;
  p.max_pieces = sp.max_pieces;
  p.ts_mul = 1.0f / short_zs_mul(W);
  p.one = 1u;
  p.zero = 0u;
  switch (W->fmt * 2 + (dx ? 1 : 0)) {
    case 0: return launch_short_t<kFmtNF4, false>(p, sp.grid, st);
    case 1: return launch_short_t<kFmtNF4, true>(p, sp.grid, st);
    case 2: return launch_short_t<kFmtMXFP4, false>(p, sp.grid, st);
    case 3: return launch_short_t<kFmtMXFP4, true>(p, sp.grid, st);
    case 4: return launch_short_t<kFmtNVFP4, false>(p, sp.grid, st);
    default: return launch_short_t<kFmtNVFP4, true>(p, sp.grid, st);
  }
}

// dB [E, N, r] = s dY_e^T T_e and dA [E, r, K] = s U_e^T X_e over each expert's rows.
qlora_status_t launch_wgrad(const void* X, const void* dY, const void* T, const void* U, int64_t M,
                            int64_t N, int64_t K, int r, float s, void* dA, void* dB, void* ws,
                            const WsLayout& L, const int32_t* offsets, int E, bool grouped,
                            cudaStream_t st) {
  WgradParams p{};
  const int rpad = rank_pad(r);
  const WgradPlan wp = wgrad_plan(N, K, M, E, num_sms());
  const CUtensorMapSwizzle rsw = swizzle_for_bytes(uint32_t(rpad) * 2);
  const uint64_t rows = uint64_t(M > 0 ? M : 1);
  if (!tmap_2d(&p.tm_l[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, uint64_t(N), rows,
               uint64_t(N) * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tmap_2d(&p.tm_l[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, uint64_t(K), rows,
               uint64_t(K) * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tmap_2d(&p.tm_r[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, T, uint64_t(r), rows,
               uint64_t(r) * 2, uint32_t(rpad), 64, rsw) ||
      !tmap_2d(&p.tm_r[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, U, uint64_t(r), rows,
               uint64_t(r) * 2, uint32_t(rpad), 64, rsw))
    return QLORA_ERR_CUDA;
  p.out0 = static_cast<__nv_bfloat16*>(dB);
  p.out1 = static_cast<__nv_bfloat16*>(dA);
  p.offsets = offsets;
  p.status = ws_status(ws);
  p.M = int(M);
  p.P0 = int(N);
  p.P1 = int(K);
  p.r = r;
  p.rpad = rpad;
  p.S = wp.S;
  p.tiles0 = wp.tiles0;
  p.tiles1 = wp.tiles1;
  p.E = E;
  p.s = s;
  const size_t smem = lora::smem_bytes(E);
  if (!set_smem(qlora_lora_wgrad_kernel, smem)) return QLORA_ERR_CUDA;
  const unsigned grid = unsigned(int64_t(E) * (wp.tiles0 + wp.tiles1) * wp.S);
  LaunchScope scope(grouped ? kKindGWgrad : kKindWgrad, st);
  if (launch_pdl_cluster(qlora_lora_wgrad_kernel, dim3(grid), dim3(lora::kThreads), smem, st, p,
                         unsigned(wp.S)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// ------------------------------------------------------------------------------ side stream
// One non-blocking stream per device for work that may overlap the caller's stream inside a call,
// with a ring of fork/join event pairs (re-recording an event is safe once its earlier waits have
// been enqueued).  Created on first use and kept for the life of the process.
struct SideStream {
  static constexpr int kEvents = 32;
  cudaStream_t stream = nullptr;
  cudaEvent_t fork[kEvents] = {};
  cudaEvent_t join[kEvents] = {};
  std::atomic<int> next{0};
};
SideStream g_side[kMaxDevices];
bool g_side_ok[kMaxDevices] = {false};
std::mutex g_side_mu;

SideStream* side_stream() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_side_mu);
  if (!g_side_ok[d]) {
    SideStream& ss = g_side[d];
    if (cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    for (int i = 0; i < SideStream::kEvents; ++i)
      if (cudaEventCreateWithFlags(&ss.fork[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&ss.join[i], cudaEventDisableTiming) != cudaSuccess)
        return nullptr;
    g_side_ok[d] = true;
  }
  return &g_side[d];
}

// ------------------------------------------------------------------- fixed scratch (no alloc)
// Scratch of qlora_linear_fwd_noalloc: a file-scope device array, present on every GPU that loads
// the library.  Host code must not pass the symbol itself to a kernel (on the host it names a
// stand-in, not device memory): its device address is looked up once per device.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_addr[kMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

// Device address of the scratch on the current device, or nullptr if it cannot be resolved.
void* noalloc_scratch_address() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[d]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return nullptr;
    g_noalloc_addr[d] = ptr;
  }
  return g_noalloc_addr[d];
}

}  // namespace
}  // namespace qlora

namespace qlora {
namespace {

// Workspace of the native W4A8 forward: header | Zs [M, r] | T [M, r] (when T_save is NULL) |
// quantised X [M, K] E4M3 | its scales [M, K/32] E8M0.
struct W4a8Layout {
  size_t zs, t, xq, xs, total;
};

W4a8Layout w4a8_layout(int64_t K, int64_t M, int r) {
  W4a8Layout L{};
  const size_t m = size_t(M > 0 ? M : 0);
  size_t off = kHeaderBytes;
  L.zs = off;
  off += align_up(m * size_t(r) * 2, 256);
  L.t = off;
  off += align_up(m * size_t(r) * 2, 256);
  L.xq = off;
  off += align_up(m * size_t(K), 256);
  L.xs = off;
  off += align_up(m * size_t(K / 32), 256);
  L.total = off;
  return L;
}

qlora_status_t launch_mxfp8_quant(const void* X, int64_t M, int64_t K, void* codes, void* scales,
                                  cudaStream_t st) {
  Mxfp8Params p{};
  p.x = static_cast<const __nv_bfloat16*>(X);
  p.codes = static_cast<uint8_t*>(codes);
  p.scales = static_cast<uint8_t*>(scales);
  p.blocks = (long long)(M * (K / 32));
  if (p.blocks == 0) return QLORA_OK;
  const unsigned grid = unsigned((p.blocks + 255) / 256);
  LaunchScope scope(kKindW4a8Quant, st);
  if (launch_pdl(qlora_mxfp8_quant_kernel, dim3(grid), dim3(256), 0, st, p) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status_t launch_w4a8_gemm(const qlora_weight_t* W, const void* xq, const void* xs,
                                const void* zs, const void* B, void* Y, int64_t M, int r,
                                int* status, cudaStream_t st) {
  using namespace w4a8;
  const int64_t N = W->N, K = W->K;
  W4a8Params p{};
  const uint64_t rows = uint64_t(M);
  if (!tmap_2d(&p.tm_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, uint64_t(K), rows, uint64_t(K), BK, BM,
               CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tmap_2d(&p.tm_w, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, W->codes, uint64_t(K), uint64_t(N),
               uint64_t(K / 2), BK, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tmap_2d(&p.tm_zs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, zs, uint64_t(r), rows, uint64_t(r) * 2,
               64, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tmap_2d(&p.tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, uint64_t(r), uint64_t(N),
               uint64_t(r) * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  p.xs = static_cast<const uint8_t*>(xs);
  p.wsc = static_cast<const uint8_t*>(W->scales);
  p.out = static_cast<__nv_bfloat16*>(Y);
  p.status = status;
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.rpad = rank_pad(r);
  p.num_m = int((M + BM - 1) / BM);
  p.num_n = int((N + BN - 1) / BN);
  p.num_k = int(K / BK);
  const int tiles = p.num_m * p.num_n;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  const size_t smem = smem_bytes();
  if (!set_smem(qlora_w4a8_gemm_kernel, smem)) return QLORA_ERR_CUDA;
  LaunchScope scope(kKindW4a8Gemm, st);
  if (launch_pdl(qlora_w4a8_gemm_kernel, dim3(grid), dim3(kThreads), smem, st, p) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" {

size_t qlora_workspace_size(int op, const qlora_weight_t* W, int64_t M, int r, int E) {
  if (check_weight(W) != QLORA_OK || M < 0 || !rank_ok(r)) return 0;
  if (op == QLORA_OP_FWD_W4A8) return w4a8_layout(W->K, M, r).total;
  const bool grouped = op == QLORA_OP_GROUPED_FWD || op == QLORA_OP_GROUPED_BWD;
  if (!grouped && op != QLORA_OP_FWD && op != QLORA_OP_BWD) return 0;
  if (grouped && (E < 1 || E > kMaxExperts)) return 0;
  const WsLayout L = ws_layout(W->N, W->K, M, r, op == QLORA_OP_BWD || op == QLORA_OP_GROUPED_BWD,
                               grouped ? E : 1, num_sms());
  return L.total;
}

qlora_status_t qlora_workspace_init(void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!ws || !aligned16(ws) || ws_bytes < kHeaderBytes) return QLORA_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, kHeaderBytes, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? QLORA_OK
             : QLORA_ERR_CUDA;
}

}  // extern "C"

namespace qlora {
namespace {

// An [M, ...] activation: required (and 16-byte aligned) when M > 0, may be NULL when M == 0.
bool act_ok(const void* q, int64_t M) { return M == 0 ? (q == nullptr || aligned16(q)) : ptr_ok(q); }

// Shared argument checks of the four training entry points.
qlora_status_t check_common(const qlora_weight_t* W, int64_t M, int r) {
  qlora_status_t st = check_weight(W);
  if (st != QLORA_OK) return st;
  if (M < 0 || M > (int64_t(1) << 31) - 512) return QLORA_ERR_INVALID_ARG;
  if (!rank_ok(r)) return (r > 0 && r <= 256) ? QLORA_ERR_UNSUPPORTED : QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}

// Forward over E experts (offsets == nullptr: one layer of M rows).
qlora_status_t run_fwd(const qlora_weight_t* W, int E, const int32_t* offsets, bool grouped,
                       const void* X, const void* A, const void* B, void* Y, void* T_save,
                       int64_t M, int r, float scale, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (!act_ok(X, M) || !ptr_ok(A) || !ptr_ok(B) || !act_ok(Y, M) || (T_save && !aligned16(T_save)))
    return QLORA_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(W->N, W->K, M, r, false, E, num_sms());
  // The split partials are optional: without room for them the tiled kernels run (so that a
  // workspace sized for a larger batch serves every smaller one).
  if (!ws || !aligned16(ws) || ws_bytes < L.partial) return QLORA_ERR_WORKSPACE;
  if (M == 0) return QLORA_OK;
  uint8_t* w = static_cast<uint8_t*>(ws);
  void* T = T_save ? T_save : w + L.t;
  void* Zs = w + L.zs;
  const float* ts = W->fmt == QLORA_FMT_NVFP4 ? W->tensor_scale : nullptr;
  float* part = reinterpret_cast<float*>(w + L.partial);
  const size_t region = ws_bytes - L.partial;
  const bool short_fwd = short_fits(W, M, E, false, region);
  const bool stream_fwd = !short_fwd && stream_fits(W, M, E, false, region);
  qlora_status_t st = launch_lora_down(false, X, M, W->K, A, r, scale, ts, T, Zs, ws_status(ws),
                                       offsets, E, grouped,
                                       (short_fwd || stream_fwd) ? kDownCtasBesideStream
                                                                 : kDownCtasBesidePair,
                                       s, short_fwd ? short_zs_mul(W) : 1.0f);
  if (st != QLORA_OK) return st;
  if (short_fwd) return launch_short(W, false, X, Zs, B, Y, M, r, ws, part, region, s);
  if (stream_fwd) return launch_stream(W, false, X, Zs, B, Y, M, r, ws_status(ws), part, region, s);
  return launch_fused(W, false, X, Zs, B, Y, M, r, ws_status(ws), offsets, E, grouped, s);
}

// Backward over E experts (offsets == nullptr: one layer of M rows).
qlora_status_t run_bwd(const qlora_weight_t* W, int E, const int32_t* offsets, bool grouped,
                       const void* X, const void* A, const void* B, const void* T, const void* dY,
                       void* dX, void* dA, void* dB, int64_t M, int r, float scale, void* ws,
                       size_t ws_bytes, cudaStream_t s) {
  if (!act_ok(X, M) || !ptr_ok(A) || !ptr_ok(B) || !act_ok(dY, M) || !ptr_ok(dA) || !ptr_ok(dB) ||
      (T && !aligned16(T)) || (dX && !aligned16(dX)))
    return QLORA_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(W->N, W->K, M, r, true, E, num_sms());
  if (!ws || !aligned16(ws) || ws_bytes < L.partial) return QLORA_ERR_WORKSPACE;   // as run_fwd
  if (M == 0) {
    if (cudaMemsetAsync(dA, 0, size_t(E) * r * W->K * 2, s) != cudaSuccess ||
        cudaMemsetAsync(dB, 0, size_t(E) * W->N * r * 2, s) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  const float* ts = W->fmt == QLORA_FMT_NVFP4 ? W->tensor_scale : nullptr;
  void* Zs = w + L.zs;
  void* U = w + L.u;
  float* part = reinterpret_cast<float*>(w + L.partial);
  const size_t region = ws_bytes - L.partial;
  qlora_status_t st;
  if (!T) {  // recompute T = X A^T (its scaled copy lands in Zs and is overwritten below) with
             // the forward's split plan, so it equals the forward's T bit for bit
    const bool beside = short_fits(W, M, E, false, region) || stream_fits(W, M, E, false, region);
    st = launch_lora_down(false, X, M, W->K, A, r, scale, ts, w + L.t, Zs, ws_status(ws), offsets,
                          E, grouped, beside ? kDownCtasBesideStream : kDownCtasBesidePair, s);
    if (st != QLORA_OK) return st;
    T = w + L.t;
  }
  const bool short_dx = dX && short_fits(W, M, E, true, region);
  const bool stream_dx = dX && !short_dx && stream_fits(W, M, E, true, region);
  st = launch_lora_down(true, dY, M, W->N, B, r, scale, ts, U, Zs, ws_status(ws), offsets, E,
                        grouped,
                        !dX ? 0 : ((short_dx || stream_dx) ? kDownCtasBesideStream : kDownCtasBesidePair),
                        s, short_dx ? short_zs_mul(W) : 1.0f, short_dx ? kDownWideCtas : 0,
                        w + L.dsum, ws);
  if (st != QLORA_OK) return st;
  auto run_dx = [&]() {
    if (short_dx) return launch_short(W, true, dY, Zs, A, dX, M, r, ws, part, region, s);
    if (stream_dx) return launch_stream(W, true, dY, Zs, A, dX, M, r, ws_status(ws), part, region, s);
    return launch_fused(W, true, dY, Zs, A, dX, M, r, ws_status(ws), offsets, E, grouped, s);
  };
  if (dX) {
    // The adapter gradients need only T, U, X and dY, so they run on a side stream beside the dX
    // kernel, on the SMs it leaves idle (the tiled kernel's last wave of tiles; the SMs the
    // streaming kernel leaves to lora_down); the kernels share no workspace region.  Joined back
    // into `s` before returning.
    SideStream* side = side_stream();
    if (side) {
      const int slot = side->next.fetch_add(1, std::memory_order_relaxed) % SideStream::kEvents;
      if (cudaEventRecord(side->fork[slot], s) != cudaSuccess ||
          cudaStreamWaitEvent(side->stream, side->fork[slot], 0) != cudaSuccess)
        return QLORA_ERR_CUDA;
      st = launch_wgrad(X, dY, T, U, M, W->N, W->K, r, scale, dA, dB, ws, L, offsets, E, grouped,
                        side->stream);
      if (st != QLORA_OK) return st;
      if (cudaEventRecord(side->join[slot], side->stream) != cudaSuccess) return QLORA_ERR_CUDA;
      st = run_dx();
      if (cudaStreamWaitEvent(s, side->join[slot], 0) != cudaSuccess) return QLORA_ERR_CUDA;
      return st;
    }
  }
  if (dX) {
    st = run_dx();
    if (st != QLORA_OK) return st;
  }
  return launch_wgrad(X, dY, T, U, M, W->N, W->K, r, scale, dA, dB, ws, L, offsets, E, grouped, s);
}

qlora_status_t check_groups(int E, const int32_t* d_offsets) {
  if (E < 1 || E > kMaxExperts) return QLORA_ERR_UNSUPPORTED;
  if (!d_offsets || (reinterpret_cast<uintptr_t>(d_offsets) & 3u) != 0) return QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}

}  // namespace
}  // namespace qlora

extern "C" {

qlora_status_t qlora_linear_fwd(const qlora_weight_t* W, const void* X, const void* A,
                                const void* B, void* Y, void* T_save, int64_t M, int r,
                                float scale, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  const qlora_status_t st = check_common(W, M, r);
  if (st != QLORA_OK) return st;
  return run_fwd(W, 1, nullptr, false, X, A, B, Y, T_save, M, r, scale, ws, ws_bytes,
                 reinterpret_cast<cudaStream_t>(stream));
}

qlora_status_t qlora_mxfp8_quantize(const void* X, int64_t M, int64_t K, void* codes, void* scales,
                                    qlora_stream_t stream) {
  if (M < 0 || K <= 0 || K % 128 != 0 || M > (int64_t(1) << 31) - 512) return QLORA_ERR_INVALID_ARG;
  if (M > 0 && (!ptr_ok(X) || !ptr_ok(codes) || !ptr_ok(scales))) return QLORA_ERR_INVALID_ARG;
  return launch_mxfp8_quant(X, M, K, codes, scales, reinterpret_cast<cudaStream_t>(stream));
}

qlora_status_t qlora_linear_fwd_w4a8(const qlora_weight_t* W, const void* X, const void* A,
                                     const void* B, void* Y, void* T_save, int64_t M, int r,
                                     float scale, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  qlora_status_t st = check_common(W, M, r);
  if (st != QLORA_OK) return st;
  if (W->fmt != QLORA_FMT_MXFP4 || W->K % 128 != 0) return QLORA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(W->codes) & 31u) != 0 || !act_ok(X, M) || !ptr_ok(A) ||
      !ptr_ok(B) || !act_ok(Y, M) || (T_save && !aligned16(T_save)))
    return QLORA_ERR_INVALID_ARG;
  const W4a8Layout L = w4a8_layout(W->K, M, r);
  if (!ws || !aligned16(ws) || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  if (M == 0) return QLORA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  void* T = T_save ? T_save : w + L.t;
  st = launch_mxfp8_quant(X, M, W->K, w + L.xq, w + L.xs, s);
  if (st != QLORA_OK) return st;
  // T = X A^T from the bf16 X and Zs = bf16(s T), as in the bf16 forward
  st = launch_lora_down(false, X, M, W->K, A, r, scale, nullptr, T, w + L.zs, ws_status(ws),
                        nullptr, 1, false, kDownCtasBesidePair, s);
  if (st != QLORA_OK) return st;
  return launch_w4a8_gemm(W, w + L.xq, w + L.xs, w + L.zs, B, Y, M, r, ws_status(ws), s);
}

qlora_status_t qlora_linear_fwd_noalloc(const qlora_weight_t* W, const void* X, const void* A,
                                        const void* B, void* Y, void* T_save, int64_t M, int r,
                                        float scale, qlora_stream_t stream) {
  qlora_status_t st = check_common(W, M, r);
  if (st != QLORA_OK) return st;
  if (!act_ok(X, M) || !ptr_ok(A) || !ptr_ok(B) || !act_ok(Y, M) || (T_save && !aligned16(T_save)))
    return QLORA_ERR_INVALID_ARG;
  const size_t mr = align_up(size_t(M) * size_t(r) * 2, 256);
  const size_t need = kNoAllocHeaderBytes + mr + (T_save ? 0 : mr);
  if (need > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;
  if (M == 0) return QLORA_OK;
  uint8_t* w = static_cast<uint8_t*>(noalloc_scratch_address());
  if (!w) return QLORA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(w, 0, kNoAllocHeaderBytes, s) != cudaSuccess) return QLORA_ERR_CUDA;
  int* status = reinterpret_cast<int*>(w);
  void* Zs = w + kNoAllocHeaderBytes;
  void* T = T_save ? T_save : w + kNoAllocHeaderBytes + mr;
  const float* ts = W->fmt == QLORA_FMT_NVFP4 ? W->tensor_scale : nullptr;
  st = launch_lora_down(false, X, M, W->K, A, r, scale, ts, T, Zs, status, nullptr, 1, false,
                        kDownCtasBesidePair, s);
  if (st != QLORA_OK) return st;
  return launch_fused(W, false, X, Zs, B, Y, M, r, status, nullptr, 1, false, s);
}

qlora_status_t qlora_linear_fwd_noalloc_status(qlora_stream_t stream) {
  uint8_t* w = static_cast<uint8_t*>(noalloc_scratch_address());
  if (!w) return QLORA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, w, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return static_cast<qlora_status_t>(v);
}

qlora_status_t qlora_linear_bwd(const qlora_weight_t* W, const void* X, const void* A,
                                const void* B, const void* T, const void* dY, void* dX, void* dA,
                                void* dB, int64_t M, int r, float scale, void* ws, size_t ws_bytes,
                                qlora_stream_t stream) {
  const qlora_status_t st = check_common(W, M, r);
  if (st != QLORA_OK) return st;
  return run_bwd(W, 1, nullptr, false, X, A, B, T, dY, dX, dA, dB, M, r, scale, ws, ws_bytes,
                 reinterpret_cast<cudaStream_t>(stream));
}

qlora_status_t qlora_grouped_fwd(const qlora_weight_t* W, int E, const int32_t* d_offsets,
                                 int64_t M_total, const void* X, const void* A, const void* B,
                                 void* Y, void* T_save, int r, float scale, void* ws,
                                 size_t ws_bytes, qlora_stream_t stream) {
  qlora_status_t st = check_common(W, M_total, r);
  if (st != QLORA_OK) return st;
  if ((st = check_groups(E, d_offsets)) != QLORA_OK) return st;
  return run_fwd(W, E, d_offsets, true, X, A, B, Y, T_save, M_total, r, scale, ws, ws_bytes,
                 reinterpret_cast<cudaStream_t>(stream));
}

qlora_status_t qlora_grouped_bwd(const qlora_weight_t* W, int E, const int32_t* d_offsets,
                                 int64_t M_total, const void* X, const void* A, const void* B,
                                 const void* T, const void* dY, void* dX, void* dA, void* dB,
                                 int r, float scale, void* ws, size_t ws_bytes,
                                 qlora_stream_t stream) {
  qlora_status_t st = check_common(W, M_total, r);
  if (st != QLORA_OK) return st;
  if ((st = check_groups(E, d_offsets)) != QLORA_OK) return st;
  return run_bwd(W, E, d_offsets, true, X, A, B, T, dY, dX, dA, dB, M_total, r, scale, ws,
                 ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

qlora_status_t qlora_get_device_status(void* ws, qlora_stream_t stream) {
  if (!ws || !aligned16(ws)) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return static_cast<qlora_status_t>(v);
}

qlora_status_t qlora_debug_dequant(const qlora_weight_t* W, int transposed, void* out,
                                   qlora_stream_t stream) {
  qlora_status_t st = check_weight(W);
  if (st != QLORA_OK) return st;
  if (!ptr_ok(out)) return QLORA_ERR_INVALID_ARG;
  if (transposed < 0 || transposed > 3) return QLORA_ERR_INVALID_ARG;
  if (transposed >= 2) {   // the short-batch kernels' decoders
    if (W->fmt == QLORA_FMT_NF4_DQ) return QLORA_ERR_UNSUPPORTED;
    ShortParams sp{};
    sp.codes = static_cast<const uint8_t*>(W->codes);
    sp.scales = W->scales;
    sp.out = static_cast<__nv_bfloat16*>(out);
    sp.N = int(W->N);
    sp.K = int(W->K);
    sp.one = 1u;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const unsigned grid = unsigned((W->N * (W->K / 64) + 127) / 128);
    const bool regs = transposed == 2;
    switch (W->fmt * 2 + (regs ? 1 : 0)) {
      case 0: qlora_debug_short_decode_kernel<kFmtNF4, false><<<grid, 128, 0, s>>>(sp); break;
      case 1: qlora_debug_short_decode_kernel<kFmtNF4, true><<<grid, 128, 0, s>>>(sp); break;
      case 2: qlora_debug_short_decode_kernel<kFmtMXFP4, false><<<grid, 128, 0, s>>>(sp); break;
      case 3: qlora_debug_short_decode_kernel<kFmtMXFP4, true><<<grid, 128, 0, s>>>(sp); break;
      case 4: qlora_debug_short_decode_kernel<kFmtNVFP4, false><<<grid, 128, 0, s>>>(sp); break;
      default: qlora_debug_short_decode_kernel<kFmtNVFP4, true><<<grid, 128, 0, s>>>(sp); break;
    }
    return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  }
  DebugDequantParams p{};
  const bool dx = transposed != 0;
  const int64_t N = W->N, K = W->K;
  if (!tmap_2d(&p.tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, uint64_t(K / 2), uint64_t(N),
               uint64_t(K / 2), dx ? 64 : 32, dx ? 64 : 128,
               dx ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B))
    return QLORA_ERR_CUDA;
  p.scales = W->scales;
  p.scales2 = W->fmt == QLORA_FMT_NF4_DQ ? W->scales2 : nullptr;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = nullptr;
  p.N = int(N);
  p.K = int(K);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid = dx ? dim3(unsigned((K + 127) / 128), unsigned((N + 63) / 64))
                       : dim3(unsigned((N + 127) / 128), unsigned(K / 64));
  switch (W->fmt * 2 + (dx ? 1 : 0)) {
    case 0: qlora_debug_dequant_kernel<kFmtNF4, false><<<grid, 128, 0, s>>>(p); break;
    case 1: qlora_debug_dequant_kernel<kFmtNF4, true><<<grid, 128, 0, s>>>(p); break;
    case 2: qlora_debug_dequant_kernel<kFmtMXFP4, false><<<grid, 128, 0, s>>>(p); break;
    case 3: qlora_debug_dequant_kernel<kFmtMXFP4, true><<<grid, 128, 0, s>>>(p); break;
    case 4: qlora_debug_dequant_kernel<kFmtNVFP4, false><<<grid, 128, 0, s>>>(p); break;
    case 5: qlora_debug_dequant_kernel<kFmtNVFP4, true><<<grid, 128, 0, s>>>(p); break;
    case 6: qlora_debug_dequant_kernel<kFmtNF4DQ, false><<<grid, 128, 0, s>>>(p); break;
    default: qlora_debug_dequant_kernel<kFmtNF4DQ, true><<<grid, 128, 0, s>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status_t qlora_quantize(const qlora_weight_t* W, const void* v, int v_is_bf16,
                              qlora_stream_t stream) {
  const qlora_status_t st = check_weight(W);
  if (st != QLORA_OK) return st;
  if (!ptr_ok(v)) return QLORA_ERR_INVALID_ARG;
  if (W->fmt == QLORA_FMT_NF4_DQ && W->N * (W->K / 64) > (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  QuantParams p{};
  p.v = v;
  p.v_bf16 = v_is_bf16 ? 1 : 0;
  p.codes = const_cast<uint8_t*>(W->codes);
  p.scales = const_cast<void*>(W->scales);
  p.scales2 = const_cast<float*>(W->scales2);
  p.tensor_scale = const_cast<float*>(W->tensor_scale);
  p.N = int(W->N);
  p.K = int(W->K);
  const int bs = quant::block_size(W->fmt == QLORA_FMT_NF4 ? kFmtNF4
                                   : W->fmt == QLORA_FMT_MXFP4 ? kFmtMXFP4
                                   : W->fmt == QLORA_FMT_NVFP4 ? kFmtNVFP4 : kFmtNF4DQ);
  const int64_t blocks = W->N * (W->K / bs);
  const unsigned grid = unsigned((blocks + quant::kBlocksPerCta - 1) / quant::kBlocksPerCta);
  if (W->fmt == QLORA_FMT_NVFP4) {
    if (cudaMemsetAsync(p.tensor_scale, 0, sizeof(float), s) != cudaSuccess) return QLORA_ERR_CUDA;
    qlora_quant_amax_kernel<<<unsigned(8 * num_sms()), 256, 0, s>>>(
        p, reinterpret_cast<unsigned*>(p.tensor_scale));
  }
  switch (W->fmt) {
    case QLORA_FMT_NF4: qlora_quant_encode_kernel<kFmtNF4><<<grid, quant::kBlocksPerCta, 0, s>>>(p); break;
    case QLORA_FMT_MXFP4: qlora_quant_encode_kernel<kFmtMXFP4><<<grid, quant::kBlocksPerCta, 0, s>>>(p); break;
    case QLORA_FMT_NVFP4: qlora_quant_encode_kernel<kFmtNVFP4><<<grid, quant::kBlocksPerCta, 0, s>>>(p); break;
    default: qlora_quant_encode_kernel<kFmtNF4DQ><<<grid, quant::kBlocksPerCta, 0, s>>>(p); break;
  }
  if (W->fmt == QLORA_FMT_NVFP4) qlora_quant_tensor_scale_kernel<<<1, 1, 0, s>>>(p.tensor_scale);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status_t qlora_merge_requantize(const qlora_weight_t* W, const void* A, const void* B, int r,
                                      float scale, const qlora_weight_t* W_out, float* merged,
                                      qlora_stream_t stream) {
  qlora_status_t st = check_weight(W);
  if (st != QLORA_OK) return st;
  st = check_weight(W_out);
  if (st != QLORA_OK) return st;
  if (W_out->N != W->N || W_out->K != W->K || r < 1 || r > 1024 || !ptr_ok(A) || !ptr_ok(B) ||
      !ptr_ok(merged))
    return QLORA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MergeParams p{};
  p.w = StoredView{W->codes, W->scales, W->scales2, W->tensor_scale, int(W->K)};
  p.A = static_cast<const __nv_bfloat16*>(A);
  p.B = static_cast<const __nv_bfloat16*>(B);
  p.out = merged;
  p.N = int(W->N);
  p.K = int(W->K);
  p.r = r;
  p.s = scale;
  const unsigned grid = unsigned(4 * num_sms());
  switch (W->fmt) {
    case QLORA_FMT_NF4: qlora_merge_values_kernel<kFmtNF4><<<grid, 256, 0, s>>>(p); break;
    case QLORA_FMT_MXFP4: qlora_merge_values_kernel<kFmtMXFP4><<<grid, 256, 0, s>>>(p); break;
    case QLORA_FMT_NVFP4: qlora_merge_values_kernel<kFmtNVFP4><<<grid, 256, 0, s>>>(p); break;
    default: qlora_merge_values_kernel<kFmtNF4DQ><<<grid, 256, 0, s>>>(p); break;
  }
  if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
  return qlora_quantize(W_out, merged, 0, stream);
}

}  // extern "C"

namespace {
// ------------------------------------------------------------------------------------- LoftQ
// Split of a tall-product's reduction: up to 296 CTAs, one wave of a 148-SM part at the GEMM's
// two CTAs per SM (a constant, so that the workspace size does not depend on the device), at
// least 512 of the reduction per split.
constexpr int64_t kLoftqTargetCtas = 296;

int loftq_splits(int64_t M, int64_t Nn, int64_t Kk) {
  const int64_t tiles = ((M + loftq::kBM - 1) / loftq::kBM) * ((Nn + loftq::kBN - 1) / loftq::kBN);
  int64_t z = kLoftqTargetCtas / tiles;   // at most one wave at two CTAs per SM
  if (z > Kk / 512) z = Kk / 512;
  if (z > 256) z = 256;
  return int(z < 1 ? 1 : z);
}

int loftq_width(int64_t N, int64_t K, int r) {
  int64_t l = r + loftq::kOversample;
  if (l > loftq::kMaxL) l = loftq::kMaxL;
  if (l > N) l = N;
  if (l > K) l = K;
  return int(l);
}

struct LoftqLayout {
  size_t R, Y, Y2, Z, Z2, omega, part, G, Mx, Cb, Ca, sig, Bf, Af, norm, total;
};

LoftqLayout loftq_layout(int64_t N, int64_t K, int r) {
  const int64_t l = loftq_width(N, K, r);
  int64_t part = 0;
  auto need = [&](int64_t M, int64_t Nn, int64_t Kk, bool always) {
    const int z = loftq_splits(M, Nn, Kk);
    if (z > 1 || always) part = std::max(part, int64_t(z) * M * Nn);
  };
  need(N, l, K, false);   // Y = R Omega, Y = R Z
  need(K, l, N, false);   // Z = R^T Y
  need(l, l, N, true);    // Y^T Y
  need(l, l, K, true);    // Z^T Z
  LoftqLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  L.R = take(size_t(N) * K * 4);
  L.Y = take(size_t(N) * l * 4);
  L.Y2 = take(size_t(N) * l * 4);
  L.Z = take(size_t(K) * l * 4);
  L.Z2 = take(size_t(K) * l * 4);
  L.omega = take(size_t(K) * l * 4);
  L.part = take(size_t(part) * 4);
  L.G = take(size_t(l) * l * 8);
  L.Mx = take(size_t(l) * l * 4);
  L.Cb = take(size_t(l) * r * 4);
  L.Ca = take(size_t(r) * l * 4);
  L.sig = take(size_t(r) * 4);
  L.Bf = take(size_t(N) * r * 4);
  L.Af = take(size_t(r) * K * 4);
  L.norm = take(size_t(loftq::kNormBlocks) * 8);
  L.total = off;
  return L;
}

// C = opA(A) opB(B) [M, Nn] (dense, ldc = Nn when split); out64: the result as fp64 instead.
template <bool TA, bool TB>
void loftq_gemm(const float* A, int64_t lda, const float* B, int64_t ldb, float* C, int64_t ldc,
                int M, int Nn, int64_t Kk, float* part, double* out64, cudaStream_t s) {
  const int z = loftq_splits(M, Nn, Kk);
  const dim3 grid(unsigned((M + loftq::kBM - 1) / loftq::kBM),
                  unsigned((Nn + loftq::kBN - 1) / loftq::kBN), unsigned(z));
  if (z == 1 && !out64) {
    loftq_gemm_kernel<TA, TB><<<grid, 256, 0, s>>>(A, lda, B, ldb, C, ldc, 0, M, Nn, Kk, Kk);
    return;
  }
  const int64_t kchunk = ((Kk + z - 1) / z + loftq::kBK - 1) / loftq::kBK * loftq::kBK;
  const int64_t count = int64_t(M) * Nn;
  loftq_gemm_kernel<TA, TB><<<grid, 256, 0, s>>>(A, lda, B, ldb, part, Nn, count, M, Nn, Kk, kchunk);
  const unsigned rb = unsigned(std::min<int64_t>((count + 255) / 256, 1184));
  loftq_reduce_kernel<<<rb, 256, 0, s>>>(part, count, z, count, out64 ? nullptr : C, out64);
}

struct LoftqRun {
  const LoftqLayout& L;
  char* ws;
  int64_t N, K;
  int r, l;
  float s;
  cudaStream_t st;
  template <typename T>
  T* at(size_t off) const { return reinterpret_cast<T*>(ws + off); }

  void jacobi(int mode) const {
    JacobiParams p{};
    p.G = at<double>(L.G);
    p.l = l;
    p.mode = mode;
    p.M = at<float>(L.Mx);
    p.Cb = at<float>(L.Cb);
    p.Ca = at<float>(L.Ca);
    p.sigma = at<float>(L.sig);
    p.r = r;
    p.s = s;
    loftq_jacobi_kernel<<<1, loftq::kJacobiThreads, loftq::jacobi_smem(l), st>>>(p);
  }
  // X [rows, l] <- a basis of its column space; X and X2 swap.  orthonormal: two SVQB passes
  // (orthonormal to fp32 precision, rank deficiency dropped: the basis Rayleigh-Ritz uses);
  // otherwise one shifted Cholesky QR step (a well-conditioned intermediate basis).
  void orth(float*& X, float*& X2, int64_t rows, bool orthonormal) const {
    for (int pass = 0; pass < (orthonormal ? 2 : 1); ++pass) {
      loftq_gemm<true, false>(X, l, X, l, nullptr, l, l, l, rows, at<float>(L.part),
                              at<double>(L.G), st);
      if (orthonormal)
        jacobi(0);
      else
        loftq_chol_kernel<<<1, loftq::kJacobiThreads, loftq::chol_smem(l), st>>>(
            at<double>(L.G), l, at<float>(L.Mx));
      loftq_gemm<false, false>(X, l, at<float>(L.Mx), l, X2, l, int(rows), l, l, nullptr, nullptr,
                               st);
      std::swap(X, X2);
    }
  }
  // Top-r SVD of R [N, K] into Bf [N, r], Af [r, K] (s Bf Af = U_r S_r V_r^T), sigma [r].
  void svd(int power_iters) const {
    const float* R = at<float>(L.R);
    float* Y = at<float>(L.Y);
    float* Y2 = at<float>(L.Y2);
    float* Z = at<float>(L.Z);
    float* Z2 = at<float>(L.Z2);
    float* part = at<float>(L.part);
    loftq_gemm<false, false>(R, K, at<float>(L.omega), l, Y, l, int(N), l, K, part, nullptr, st);
    orth(Y, Y2, N, power_iters == 0);
    for (int q = 0; q < power_iters; ++q) {
      loftq_gemm<true, false>(R, K, Y, l, Z, l, int(K), l, N, part, nullptr, st);
      orth(Z, Z2, K, false);
      loftq_gemm<false, false>(R, K, Z, l, Y, l, int(N), l, K, part, nullptr, st);
      orth(Y, Y2, N, q + 1 == power_iters);
    }
    loftq_gemm<true, false>(R, K, Y, l, Z, l, int(K), l, N, part, nullptr, st);
    loftq_gemm<true, false>(Z, l, Z, l, nullptr, l, l, l, K, part, at<double>(L.G), st);
    jacobi(1);
    loftq_gemm<false, false>(Y, l, at<float>(L.Cb), r, at<float>(L.Bf), r, int(N), r, l, nullptr,
                             nullptr, st);
    loftq_gemm<false, true>(at<float>(L.Ca), l, Z, l, at<float>(L.Af), K, r, int(K), l, nullptr,
                            nullptr, st);
  }
};

void loftq_residual(const qlora_weight_t* Q, const float* W, float* R, double* part, cudaStream_t s) {
  const StoredView v{Q->codes, Q->scales, Q->scales2, Q->tensor_scale, int(Q->K)};
  const int N = int(Q->N), K = int(Q->K);
  const unsigned g = loftq::kNormBlocks;
  switch (Q->fmt) {
    case QLORA_FMT_NF4: loftq_residual_kernel<kFmtNF4><<<g, 256, 0, s>>>(W, v, R, N, K, part); break;
    case QLORA_FMT_MXFP4: loftq_residual_kernel<kFmtMXFP4><<<g, 256, 0, s>>>(W, v, R, N, K, part); break;
    case QLORA_FMT_NVFP4: loftq_residual_kernel<kFmtNVFP4><<<g, 256, 0, s>>>(W, v, R, N, K, part); break;
    default: loftq_residual_kernel<kFmtNF4DQ><<<g, 256, 0, s>>>(W, v, R, N, K, part); break;
  }
}
}  // namespace

extern "C" {

size_t qlora_loftq_workspace_size(int64_t N, int64_t K, int r) {
  if (N < 1 || K < 1 || r < 1 || r > loftq::kMaxL || r > N || r > K) return 0;
  return loftq_layout(N, K, r).total;
}

qlora_status_t qlora_loftq(const float* W, const qlora_weight_t* Q, int r, float scale, int iters,
                           int power_iters, uint64_t seed, void* A_out, void* B_out, float* errs,
                           float* sigma, void* work, size_t work_bytes, qlora_stream_t stream) {
  qlora_status_t st = check_weight(Q);
  if (st != QLORA_OK) return st;
  const int64_t N = Q->N, K = Q->K;
  if (r < 1 || r > loftq::kMaxL || r > N || r > K || !(scale > 0.0f) || !(scale < 3.0e38f) ||
      iters < 1 || iters > 64 || power_iters < 0 || power_iters > 16 || !ptr_ok(W) ||
      !ptr_ok(A_out) || !ptr_ok(B_out) || !errs || (reinterpret_cast<uintptr_t>(errs) & 3u) ||
      (sigma && (reinterpret_cast<uintptr_t>(sigma) & 3u)) || !work ||
      (reinterpret_cast<uintptr_t>(work) & 255u) || N * K > (int64_t(1) << 31))
    return QLORA_ERR_INVALID_ARG;
  const LoftqLayout L = loftq_layout(N, K, r);
  if (work_bytes < L.total) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!set_smem(loftq_jacobi_kernel, loftq::jacobi_smem(loftq::kMaxL)) ||
      !set_smem(loftq_chol_kernel, loftq::chol_smem(loftq::kMaxL)))
    return QLORA_ERR_CUDA;
  const LoftqRun run{L, static_cast<char*>(work), N, K, r, loftq_width(N, K, r), scale, s};
  float* R = run.at<float>(L.R);
  double* norm = run.at<double>(L.norm);
  const int64_t n_omega = K * run.l;
  loftq_omega_kernel<<<unsigned(std::min<int64_t>((n_omega + 255) / 256, 1184)), 256, 0, s>>>(
      run.at<float>(L.omega), n_omega, seed);
  st = qlora_quantize(Q, W, 0, stream);                     // Q_1 = quantise(W)
  if (st != QLORA_OK) return st;
  for (int t = 1; t <= iters; ++t) {
    loftq_residual(Q, W, R, norm, s);                       // R_t = W - deq(Q_t)
    if (t == 1) loftq_norm_kernel<<<1, 32, 0, s>>>(norm, loftq::kNormBlocks, errs);
    run.svd(power_iters);                                   // s B_t A_t = top-r part of R_t
    const int more = t < iters;
    loftq_shift_kernel<<<loftq::kNormBlocks, 256, 0, s>>>(W, R, run.at<float>(L.Bf),
                                                          run.at<float>(L.Af), int(N), int(K), r,
                                                          scale, more, norm);
    loftq_norm_kernel<<<1, 32, 0, s>>>(norm, loftq::kNormBlocks, errs + t);
    if (more) {
      st = qlora_quantize(Q, R, 0, stream);                 // Q_{t+1} = quantise(W - s B_t A_t)
      if (st != QLORA_OK) return st;
    }
  }
  loftq_to_bf16_kernel<<<256, 256, 0, s>>>(run.at<float>(L.Af),
                                           static_cast<__nv_bfloat16*>(A_out), int64_t(r) * K);
  loftq_to_bf16_kernel<<<256, 256, 0, s>>>(run.at<float>(L.Bf),
                                           static_cast<__nv_bfloat16*>(B_out), N * r);
  if (sigma && cudaMemcpyAsync(sigma, run.at<float>(L.sig), size_t(r) * 4,
                               cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status_t qlora_debug_decode_rate(int fmt, int iters, double* weights_per_clock_per_sm) {
  if (!weights_per_clock_per_sm || iters < 1 || iters > (1 << 20) || fmt < QLORA_FMT_NF4 ||
      fmt > QLORA_FMT_NF4_DQ)
    return QLORA_ERR_INVALID_ARG;
  if (fmt == QLORA_FMT_NF4_DQ) fmt = QLORA_FMT_NF4;   // the same item decode once the absmax is formed
  const int sms = num_sms();
  unsigned long long* cyc = nullptr;
  uint32_t* sink = nullptr;
  if (cudaMalloc(&cyc, sizeof(unsigned long long) * sms) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMalloc(&sink, 4) != cudaSuccess) {
    cudaFree(cyc);
    return QLORA_ERR_CUDA;
  }
  if (fmt == QLORA_FMT_NF4) qlora_debug_decode_rate_kernel<kFmtNF4><<<sms, 512>>>(iters, cyc, sink, 1u);
  else if (fmt == QLORA_FMT_MXFP4) qlora_debug_decode_rate_kernel<kFmtMXFP4><<<sms, 512>>>(iters, cyc, sink, 1u);
  else qlora_debug_decode_rate_kernel<kFmtNVFP4><<<sms, 512>>>(iters, cyc, sink, 1u);
  std::vector<unsigned long long> h(sms);
  const bool ok = cudaGetLastError() == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess &&
                  cudaMemcpy(h.data(), cyc, sizeof(unsigned long long) * sms,
                             cudaMemcpyDeviceToHost) == cudaSuccess;
  cudaFree(cyc);
  cudaFree(sink);
  if (!ok) return QLORA_ERR_CUDA;
  double c = 0;
  for (int i = 0; i < sms; ++i) c += double(h[i]);
  c /= sms;
  *weights_per_clock_per_sm = c > 0 ? double(iters) * 512.0 * 64.0 / c : 0.0;
  return QLORA_OK;
}

qlora_status_t qlora_debug_wait_timeout(void* ws, size_t ws_bytes, int limit_us,
                                        qlora_stream_t stream) {
  if (!ws || !aligned16(ws) || ws_bytes < kHeaderBytes) return QLORA_ERR_WORKSPACE;
  if (limit_us <= 0 || limit_us > 1000000) return QLORA_ERR_INVALID_ARG;
  int clk_khz = 0;
  if (cudaDeviceGetAttribute(&clk_khz, cudaDevAttrClockRate, current_device()) != cudaSuccess ||
      clk_khz <= 0)
    clk_khz = 2000000;
  const unsigned long long cycles = (unsigned long long)limit_us * (unsigned long long)clk_khz / 1000ull;
  qlora_debug_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ws_status(ws), cycles);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

const char* qlora_status_string(qlora_status_t status) {
  switch (status) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument (pointer, alignment or shape)";
    case QLORA_ERR_UNSUPPORTED: return "unsupported by this build (e.g. rank not in {8,16,32,64})";
    case QLORA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case QLORA_ERR_CUDA: return "a CUDA call failed (launch or tensor map)";
    case QLORA_ERR_DEVICE_TIMEOUT: return "a device-side pipeline wait gave up";
  }
  return "unknown status";
}

#ifdef QLORA_DEBUG
const char* qlora_build_info(void) { return "qlora-b200 0.1 sm_100a debug (device bounds checks)"; }
#else
const char* qlora_build_info(void) { return "qlora-b200 0.1 sm_100a"; }
#endif

int64_t qlora_launch_count(void) { return g_launches.load(); }

qlora_status_t qlora_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (enable && g_ev.empty()) {
    g_ev.resize(2 * size_t(kMaxProfiled));
    for (auto& e : g_ev)
      if (cudaEventCreate(&e) != cudaSuccess) {
        g_ev.clear();
        return QLORA_ERR_CUDA;
      }
  }
  g_prof_on = enable != 0;
  return QLORA_OK;
}

qlora_status_t qlora_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_rec_kind.clear();
  return QLORA_OK;
}

qlora_status_t qlora_profile_read(int max_kinds, int* n_kinds, const char** names, int* counts,
                                  double* total_ms) {
  if (!n_kinds || max_kinds < 0 || (max_kinds > 0 && (!names || !counts || !total_ms)))
    return QLORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int cnt[kNumKinds] = {0};
  double ms[kNumKinds] = {0.0};
  for (size_t i = 0; i < g_rec_kind.size(); ++i) {
    if (cudaEventSynchronize(g_ev[2 * i + 1]) != cudaSuccess) return QLORA_ERR_CUDA;
    float t = 0.0f;
    if (cudaEventElapsedTime(&t, g_ev[2 * i], g_ev[2 * i + 1]) != cudaSuccess) return QLORA_ERR_CUDA;
    cnt[g_rec_kind[i]] += 1;
    ms[g_rec_kind[i]] += t;
  }
  int n = 0;
  for (int k = 0; k < kNumKinds; ++k) {
    if (cnt[k] == 0) continue;
    if (n < max_kinds) {
      names[n] = kKindNames[k];
      counts[n] = cnt[k];
      total_ms[n] = ms[k];
    }
    ++n;
  }
  *n_kinds = n;
  return QLORA_OK;
}

}  // extern "C"
