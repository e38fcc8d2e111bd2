// qlora_lora.cuh -- the rank-r side path of the layer on tcgen05.
//
// lora_down: Z[M, r] = Act[M, Kc] . R, 128-row tiles, the contraction split over S CTAs per tile.
//   forward : Z = T = X A^T   (R = A^T: A [r, K] is a K-major operand)
//   backward: Z = U = dY B    (R = B:   B [N, r] is an MN-major operand)
//   It writes Z (bf16) and Zs = bf16(Z * s / ts), the operand of the fused GEMM's LoRA step.
//   ("Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §2 "Initialization matters": z = A x
//   and dL/dz = B^T dL/dy.)
//
// lora_wgrad: the adapter gradients, reductions over the M rows:
//   dB[N, r] = s . dY^T T     and     dA^T[K, r] = s . X^T U   (dA written as [r, K])
//   ("Training LLMs on a Budget", §2 "Initialization matters": dL/dB = dL/dy z^T,
//   dL/dA = (B^T dL/dy) x^T, with the layer's scale s.)  Both are out[P, r] = s . L^T R with L
//   [M, P] and R [M, r]: an M=128 x N=rpad tcgen05 GEMM per 128-row tile of P whose operands are
//   both MN-major (M is the contraction), M split over S CTAs per tile.
//
// Grouped launches (expert e owns rows [off[e], off[e+1]) of the packed activations, with its own
// adapters) run the same kernels over a device-side table of (expert, tile) built from the
// offsets; a single layer is one expert.  lora_down computes rows beyond an expert's end with
// that expert's adapter and drops them at the store; lora_wgrad zeroes them in shared memory
// before the MMA, so no row of another expert enters a reduction.
//
// Both kernels are memory bound (they stream an activation once) and have few output tiles, so
// the contraction is split over S CTAs per tile to fill the GPU.  The S CTAs of a tile run as one
// thread-block cluster and add their fp32 partial tiles through distributed shared memory, in
// split order 0..S-1, so the result is bitwise deterministic.  A short batch (one tile) has too
// few splits for that: lora_down may then run C clusters per tile over consecutive ranges of the
// contraction; each cluster stores its sum as fp32 in the workspace and the last cluster to
// arrive (an arrival counter per row slice, reset by that cluster) adds the C sums in cluster
// order 0..C-1, again a fixed order.
#pragma once
#include <cuda_bf16.h>
#include "qlora_ptx.cuh"
#include "qlora_groups.cuh"

namespace qlora {
namespace lora {
constexpr int BM = 128, BK = 64, NS = 8;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int R_BYTES = 64 * 128;     // up to 64 x 128 B
constexpr int kThreads = 6 * 32;      // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kTmemCols = 64;
constexpr int kMaxClusters = 8;       // C > 1: the workspace holds the sums of 8 clusters of one tile
constexpr size_t kSmemBase = 1024 + size_t(NS) * (A_BYTES + R_BYTES) + 512;
__host__ __device__ constexpr size_t smem_bytes(int E) { return kSmemBase + size_t(2) * (E + 1) * 4; }
}  // namespace lora

__device__ __forceinline__ uint32_t swz_mode_for_row_bytes(uint32_t rowb) {
  return rowb == 128 ? ptx::kSw128 : (rowb == 64 ? ptx::kSw64 : ptx::kSw32);
}

// Split-K reduction through distributed shared memory.  The S CTAs that share one 128-row output
// tile form a thread-block cluster (cluster rank = split).  Each stores its fp32 partial tile
// (128 rows x rpad, row-major, 16-byte chunks XOR-swizzled by row so that the row-per-lane stores
// of a warp do not conflict) in its own shared memory; after a cluster barrier, CTA `split` sums
// rows [split * ceil(128 / S), ...) of all S partials, read in split order 0..S-1 -- so the result
// is bitwise deterministic -- and a second cluster barrier keeps every partial in place until all
// reads are done.
__device__ __forceinline__ uint32_t part_off(int row, int chunk, uint32_t rowb) {
  const uint32_t sw = rowb >= 128u ? (uint32_t(row) & 7u) : ((uint32_t(row) >> 1) & 3u);
  return uint32_t(row) * rowb + ((uint32_t(chunk) ^ sw) << 4);
}

// This thread's accumulator row (rpad fp32 values) as row `lrow` of the partial tile at `part`.
__device__ __forceinline__ void store_partial_row(uint32_t part, int lrow, const float (&acc)[64],
                                                  int rpad) {
  const uint32_t rowb = uint32_t(rpad) * 4u;
#pragma unroll
  for (int c = 0; c < 16; ++c)
    if (c * 4 < rpad)
      ptx::st_shared_v4(part + part_off(lrow, c, rowb), __float_as_uint(acc[4 * c]),
                        __float_as_uint(acc[4 * c + 1]), __float_as_uint(acc[4 * c + 2]),
                        __float_as_uint(acc[4 * c + 3]));
}

// Run by the 128 epilogue threads (et = 0..127) between the two cluster barriers: rows [0, nrows)
// of the tile exist; write(row, c0, v[8]) receives the sum of columns c0 .. c0+7 of a row.
template <class F>
__device__ __forceinline__ void cluster_sum(uint32_t part, int rpad, int S, int split, int nrows,
                                            int et, F&& write) {
  const int rows_per = (lora::BM + S - 1) / S;
  const int r0 = split * rows_per;
  const int r1 = min(nrows, r0 + rows_per);
  const int g8 = rpad / 8;
  const int items = r1 > r0 ? (r1 - r0) * g8 : 0;
  const uint32_t rowb = uint32_t(rpad) * 4u;
  for (int it = et; it < items; it += 128) {
    const int lr = r0 + it / g8, c8 = it % g8;
    const uint32_t o0 = part_off(lr, 2 * c8, rowb), o1 = part_off(lr, 2 * c8 + 1, rowb);
    float v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) v[c] = 0.f;
    for (int sp = 0; sp < S; sp += 8) {
      float4 a[8], b[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (sp + q < S) {
          const uint32_t rb = ptx::mapa(part, uint32_t(sp + q));
          a[q] = ptx::ld_dsmem_f4(rb + o0);
          b[q] = ptx::ld_dsmem_f4(rb + o1);
        }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (sp + q < S) {
          v[0] += a[q].x; v[1] += a[q].y; v[2] += a[q].z; v[3] += a[q].w;
          v[4] += b[q].x; v[5] += b[q].y; v[6] += b[q].z; v[7] += b[q].w;
        }
    }
    write(lr, c8 * 8, v);
  }
}

// Load this thread's accumulator row (rpad columns) from tensor memory.
__device__ __forceinline__ void load_acc_row(uint32_t taddr, int rpad, float (&acc)[64]) {
#pragma unroll
  for (int c = 0; c < 64; c += 16) {
    if (c < rpad) {
      uint32_t v[16];
      ptx::tmem_ld_32x32b_x16(taddr + c, v);
      ptx::tmem_ld_wait(v);
#pragma unroll
      for (int g = 0; g < 16; ++g) acc[c + g] = __uint_as_float(v[g]);
    } else {
#pragma unroll
      for (int g = 0; g < 16; ++g) acc[c + g] = 0.0f;
    }
  }
}

struct DownParams {
  CUtensorMap tm_act;  // X [M, K] or dY [M, N] bf16, box {64, 128}, SW128
  CUtensorMap tm_r;    // T: A [E, r, K] box {64, rpad, 1} SW128; U: B [E, N, r] box {rpad, 64, 1}
  const float* tensor_scale;   // NVFP4: [E], else nullptr
  __nv_bfloat16* z;    // [M, r]
  __nv_bfloat16* zs;   // [M, r]
  const int32_t* offsets;      // grouped: device [E+1]; nullptr: one expert
  int* status;
  float* cpart;        // C > 1: the clusters' sums [tiles][C][128][rpad] fp32
  unsigned* ccount;    // C > 1: arrival counters [tiles][S], zero between launches
  int M, r, rpad, num_k, S, C, steps_per_split, E;
  float s;
  float zs_mul;        // an exact power of two folded into Zs (2^-8 when the next kernel decodes
                       // NVFP4 elements times 2^-8), else 1
};

template <bool R_MN>
__global__ void __launch_bounds__(lora::kThreads, 1)
qlora_lora_down_kernel(const __grid_constant__ DownParams p) {
  using namespace lora;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* as = smem;
  uint8_t* rs = as + NS * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(rs + NS * R_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile unsigned* s_ticket = reinterpret_cast<volatile unsigned*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(smem + (kSmemBase - 1024));
  int* s_first = s_off + (p.E + 1);
  const uint32_t b0 = ptx::smem_u32(bars);
  auto full = [&](uint32_t s) { return b0 + 8u * s; };
  auto empty = [&](uint32_t s) { return b0 + 8u * (NS + s); };
  const uint32_t acc_full = b0 + 8u * (2 * NS);

  // (expert, 128-row tile, split) of this CTA; CTAs beyond the table's last tile have no work.
  // The table's tile count and the grid are multiples of S, so the S CTAs of a cluster either
  // all leave here or all stay.
  // With C clusters per tile the table repeats each tile S * C times: global split gs = cg * S +
  // split covers steps [gs * steps_per_split, ...), cluster cg of the tile holds splits
  // cg * S .. cg * S + S - 1 (consecutive CTAs, so one cluster).
  const int per_tile = p.S * p.C;
  const GroupView gv = build_group_view(p.offsets, p.E, p.M, BM, per_tile, s_off, s_first, p.status);
  if (int(blockIdx.x) >= gv.total()) return;
  const int e = gv.expert_of(blockIdx.x);
  const int local = int(blockIdx.x) - gv.first[e];
  const int mt = local / per_tile, gs = local % per_tile;
  const int split = gs % p.S, cg = gs / p.S;
  const int tidx = int(blockIdx.x) / per_tile;          // the tile's index in the table
  const int m0 = gv.off[e] + mt * BM;
  const int row_end = gv.off[e + 1];
  const int ks0 = min(gs * p.steps_per_split, p.num_k);
  const int ks1 = min(ks0 + p.steps_per_split, p.num_k);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) { ptx::mbar_init(full(s), 1); ptx::mbar_init(empty(s), 1); }
    ptx::mbar_init(acc_full, 1);
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const uint32_t rowb = uint32_t(p.rpad) * 2u;
  const uint32_t r_bytes = uint32_t(p.rpad) * 128u;
  const float ts = p.tensor_scale ? __ldg(p.tensor_scale + e) : 1.0f;
  const float zscale = p.s / ts * p.zs_mul;
  // Z and Zs = bf16(Z * s / ts) for columns c .. c+7 of row rw
  auto write8 = [&](int rw, int c, const float (&v)[8]) {
    if (c >= p.r) return;
    if (!ptx::dcheck(rw >= 0 && rw < p.M, p.status)) return;
    uint4 z, zs;
    z.x = ptx::cvt_bf16x2(v[0], v[1]); z.y = ptx::cvt_bf16x2(v[2], v[3]);
    z.z = ptx::cvt_bf16x2(v[4], v[5]); z.w = ptx::cvt_bf16x2(v[6], v[7]);
    zs.x = ptx::cvt_bf16x2(v[0] * zscale, v[1] * zscale);
    zs.y = ptx::cvt_bf16x2(v[2] * zscale, v[3] * zscale);
    zs.z = ptx::cvt_bf16x2(v[4] * zscale, v[5] * zscale);
    zs.w = ptx::cvt_bf16x2(v[6] * zscale, v[7] * zscale);
    *reinterpret_cast<uint4*>(p.z + size_t(rw) * p.r + c) = z;
    *reinterpret_cast<uint4*>(p.zs + size_t(rw) * p.r + c) = zs;
  };

  if (warp == 0) {
    if (lane == 0) {
      for (int ks = ks0; ks < ks1; ++ks) {
        const int it = ks - ks0;
        const uint32_t s = it % NS, ph = (it / NS) & 1;
        if (!ptx::mbar_wait(empty(s), ph ^ 1u, p.status, abort_flag)) break;
        ptx::mbar_arrive_expect_tx(full(s), A_BYTES + r_bytes);
        if (!ptx::dcheck(ptx::tma_x_ok(ks * BK, 2) && e < p.E, p.status)) break;
        ptx::tma_load_2d(ptx::smem_u32(as + s * A_BYTES), &p.tm_act, full(s), ks * BK, m0);
        if (!R_MN) ptx::tma_load_3d(ptx::smem_u32(rs + s * R_BYTES), &p.tm_r, full(s), ks * BK, 0, e);
        else ptx::tma_load_3d(ptx::smem_u32(rs + s * R_BYTES), &p.tm_r, full(s), 0, ks * BK, e);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && ks1 > ks0) {
      const uint32_t idesc = ptx::idesc_bf16(128, uint32_t(p.rpad), 0, R_MN ? 1u : 0u);
      bool ok = true;
      for (int ks = ks0; ks < ks1; ++ks) {
        const int it = ks - ks0;
        const uint32_t s = it % NS, ph = (it / NS) & 1;
        if (!ptx::mbar_wait(full(s), ph, p.status, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t a = ptx::smem_u32(as + s * A_BYTES), b = ptx::smem_u32(rs + s * R_BYTES);
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = ptx::smem_desc(a + kk * 32, 16, 1024, ptx::kSw128);
          const uint64_t bd = R_MN ? ptx::smem_desc(b + kk * 16 * rowb, 64 * rowb, 8 * rowb,
                                                    swz_mode_for_row_bytes(rowb))
                                   : ptx::smem_desc(b + kk * 32, 16, 1024, ptx::kSw128);
          ptx::mma_bf16(tmem, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(empty(s));
      }
      if (ok) ptx::mma_commit(acc_full);
    }
  } else {
    const int q = warp & 3;
    const int row = m0 + q * 32 + lane;
    const bool have = ks1 > ks0;
    if (have) ptx::mbar_wait(acc_full, 0, p.status, abort_flag);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (*abort_flag == 0) {
      float acc[64];
      if (have) {
        ptx::tc_fence_after();
        load_acc_row(tmem + (uint32_t(q * 32) << 16), p.rpad, acc);
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] = 0.0f;
      }
      if (p.S == 1) {
        if (row < row_end) {
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = acc[c + u];
            write8(row, c, v);
          }
        }
      } else {
        // the operand stages are free: every MMA has completed and every load was consumed
        store_partial_row(ptx::smem_u32(as), q * 32 + lane, acc, p.rpad);
      }
    }
  }
  if (p.S > 1) {
    const int nrows = min(BM, row_end - m0);
    // C > 1: this cluster's sum of row lr, columns c .. c+7 (the sums of one tile's clusters and
    // its S counters are what the workspace holds)
    float* const csum = p.cpart + (size_t(tidx) * p.C + cg) * BM * p.rpad;
    const bool wide_ok = p.C == 1 || ptx::dcheck(tidx == 0 && p.C <= kMaxClusters, p.status);
    ptx::cluster_sync();
    if (warp >= 2 && *abort_flag == 0 && wide_ok) {
      if (p.C == 1)
        cluster_sum(ptx::smem_u32(as), p.rpad, p.S, split, nrows, threadIdx.x - 64,
                    [&](int lr, int c, const float (&v)[8]) { write8(m0 + lr, c, v); });
      else
        cluster_sum(ptx::smem_u32(as), p.rpad, p.S, split, nrows, threadIdx.x - 64,
                    [&](int lr, int c, const float (&v)[8]) {
                      float4* d = reinterpret_cast<float4*>(csum + size_t(lr) * p.rpad + c);
                      __stcg(d, make_float4(v[0], v[1], v[2], v[3]));
                      __stcg(d + 1, make_float4(v[4], v[5], v[6], v[7]));
                    });
    }
    ptx::cluster_sync();
    if (p.C > 1 && warp >= 2 && wide_ok) {
      // Count this cluster's slice in (also after an abort, so the counter stays consistent);
      // the last of the C clusters adds the slice's C sums in cluster order.
      const int et = int(threadIdx.x) - 64;
      unsigned* const counter = p.ccount + tidx * p.S + split;
      __threadfence();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (et == 0) *s_ticket = atomicAdd(counter, 1u);
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (*s_ticket == unsigned(p.C - 1)) {
        __threadfence();
        const int rows_per = (BM + p.S - 1) / p.S;
        const int r0 = split * rows_per, r1 = min(nrows, r0 + rows_per);
        const int g8 = p.rpad / 8;
        const int items = r1 > r0 ? (r1 - r0) * g8 : 0;
        const float* const c0 = p.cpart + size_t(tidx) * p.C * BM * p.rpad;
        for (int it = et; it < items && *abort_flag == 0; it += 128) {
          const int lr = r0 + it / g8, c = (it % g8) * 8;
          float v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = 0.0f;
          for (int k = 0; k < p.C; ++k) {
            const float4* src = reinterpret_cast<const float4*>(c0 + (size_t(k) * BM + lr) * p.rpad + c);
            const float4 a = __ldcg(src), b = __ldcg(src + 1);
            v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
            v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
          }
          write8(m0 + lr, c, v);
        }
        if (et == 0) *counter = 0u;
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
}

struct WgradParams {
  CUtensorMap tm_l[2];  // L: dY [M, N] (problem 0, dB) / X [M, K] (problem 1, dA); box {64, 64} SW128
  CUtensorMap tm_r[2];  // R: T [M, r] / U [M, r]; box {rpad, 64} SW(2 rpad)
  __nv_bfloat16* out0;  // dB [E, N, r]: (p, j) at p * r + j
  __nv_bfloat16* out1;  // dA [E, r, K]: (p, j) at j * K + p
  const int32_t* offsets;       // grouped: device [E+1]; nullptr: one expert of M rows
  int* status;
  int M, P0, P1, r, rpad, S, tiles0, tiles1, E;
  float s;
};

__global__ void __launch_bounds__(lora::kThreads, 1)
qlora_lora_wgrad_kernel(const __grid_constant__ WgradParams p) {
  using namespace lora;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* as = smem;
  uint8_t* rs = as + NS * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(rs + NS * R_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_off = reinterpret_cast<int*>(smem + (kSmemBase - 1024));
  int* s_first = s_off + (p.E + 1);
  const uint32_t b0 = ptx::smem_u32(bars);
  auto full = [&](uint32_t s) { return b0 + 8u * s; };
  auto empty = [&](uint32_t s) { return b0 + 8u * (NS + s); };
  const uint32_t acc_full = b0 + 8u * (2 * NS);

  // tile = (expert, output tile of dB or dA); the expert's rows are split into S ranges of
  // whole 64-row chunks
  const GroupView gv = build_group_view(p.offsets, p.E, p.M, 64, 1, s_off, s_first, p.status);
  const int tiles_pe = p.tiles0 + p.tiles1;
  const int tile = blockIdx.x / p.S, split = blockIdx.x % p.S;
  const int e = tile / tiles_pe, et_tile = tile - e * tiles_pe;
  const int prob = et_tile < p.tiles0 ? 0 : 1;
  const int p0 = (et_tile - (prob ? p.tiles0 : 0)) * BM;
  const int P = prob ? p.P1 : p.P0;
  const bool table_ok = gv.total() > 0 || p.M == 0;
  const int row_begin = gv.off[e], row_end = gv.off[e + 1];
  const int chunks = table_ok ? (row_end - row_begin + 63) / 64 : 0;
  const int sps = (chunks + p.S - 1) / p.S;
  const int ks0 = split * sps;
  const int ks1 = min(ks0 + sps, chunks);
  const CUtensorMap* tml = &p.tm_l[prob];
  const CUtensorMap* tmr = &p.tm_r[prob];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) { ptx::mbar_init(full(s), 1); ptx::mbar_init(empty(s), 1); }
    ptx::mbar_init(acc_full, 1);
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const uint32_t rowb = uint32_t(p.rpad) * 2u;
  const uint32_t r_bytes = 64u * rowb;
  __nv_bfloat16* out0 = p.out0 + size_t(e) * p.P0 * p.r;
  __nv_bfloat16* out1 = p.out1 + size_t(e) * p.r * p.P1;
  // s * the reduction for columns c .. c+7 of output row pr (dB row-major, dA transposed)
  auto write8 = [&](int pr, int c, const float (&v)[8]) {
    if (c >= p.r) return;
    if (!ptx::dcheck(pr >= 0 && pr < (prob == 0 ? p.P0 : p.P1) && e < p.E, p.status)) return;
    if (prob == 0) {
      uint4 o;
      o.x = ptx::cvt_bf16x2(v[0] * p.s, v[1] * p.s);
      o.y = ptx::cvt_bf16x2(v[2] * p.s, v[3] * p.s);
      o.z = ptx::cvt_bf16x2(v[4] * p.s, v[5] * p.s);
      o.w = ptx::cvt_bf16x2(v[6] * p.s, v[7] * p.s);
      *reinterpret_cast<uint4*>(out0 + size_t(pr) * p.r + c) = o;
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) out1[size_t(c + u) * p.P1 + pr] = __float2bfloat16_rn(v[u] * p.s);
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      for (int ks = ks0; ks < ks1; ++ks) {
        const int it = ks - ks0;
        const uint32_t s = it % NS, ph = (it / NS) & 1;
        if (!ptx::mbar_wait(empty(s), ph ^ 1u, p.status, abort_flag)) break;
        ptx::mbar_arrive_expect_tx(full(s), A_BYTES + r_bytes);
        const uint32_t ad = ptx::smem_u32(as + s * A_BYTES);
        const int m = row_begin + ks * BK;
        if (!ptx::dcheck(ptx::tma_x_ok(p0, 2) && m >= 0 && m < p.M, p.status)) break;
        ptx::tma_load_2d(ad, tml, full(s), p0, m);
        ptx::tma_load_2d(ad + A_BYTES / 2, tml, full(s), p0 + 64, m);
        ptx::tma_load_2d(ptx::smem_u32(rs + s * R_BYTES), tmr, full(s), 0, m);
      }
    }
  } else if (warp == 1) {
    // the whole warp runs the loop: it zeroes the rows of a chunk that lie past the expert's
    // last row (both operands) before lane 0 issues the MMAs
    if (ks1 > ks0) {
      const uint32_t idesc = ptx::idesc_bf16(128, uint32_t(p.rpad), 1u, 1u);
      const uint32_t rsw = swz_mode_for_row_bytes(rowb);
      bool ok = true;
      for (int ks = ks0; ks < ks1; ++ks) {
        const int it = ks - ks0;
        const uint32_t s = it % NS, ph = (it / NS) & 1;
        if (!ptx::mbar_wait(full(s), ph, p.status, abort_flag)) { ok = false; break; }
        const uint32_t a = ptx::smem_u32(as + s * A_BYTES), b = ptx::smem_u32(rs + s * R_BYTES);
        const int valid = row_end - (row_begin + ks * BK);
        if (valid < BK) {
          // L tile: 2 blocks x 64 rows x 128 B; R tile: 64 rows x rowb bytes
          for (int idx = lane; idx < (BK - valid) * 16; idx += 32) {
            const int rr = valid + idx / 16, c = idx % 16;
            ptx::st_shared_v4(a + (c / 8) * 8192 + rr * 128 + (c % 8) * 16, 0, 0, 0, 0);
          }
          for (int idx = lane; idx < (BK - valid) * int(rowb / 16); idx += 32) {
            const int rr = valid + idx / int(rowb / 16), c = idx % int(rowb / 16);
            ptx::st_shared_v4(b + rr * rowb + c * 16, 0, 0, 0, 0);
          }
          ptx::fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          ptx::tc_fence_after();
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = ptx::smem_desc(a + kk * 2048, 8192, 1024, ptx::kSw128);
            const uint64_t bd = ptx::smem_desc(b + kk * 16 * rowb, 64 * rowb, 8 * rowb, rsw);
            ptx::mma_bf16(tmem, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
          ptx::mma_commit(empty(s));
        }
        __syncwarp();
      }
      if (ok && lane == 0) ptx::mma_commit(acc_full);
    }
  } else {
    const int q = warp & 3;
    const int prow = p0 + q * 32 + lane;
    const bool have = ks1 > ks0;
    if (have) ptx::mbar_wait(acc_full, 0, p.status, abort_flag);
    // every epilogue thread takes the same branch below: a thread whose wait gave up set
    // abort_flag before this barrier
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (*abort_flag == 0) {
      float acc[64];
      if (have) {
        ptx::tc_fence_after();
        load_acc_row(tmem + (uint32_t(q * 32) << 16), p.rpad, acc);
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] = 0.0f;
      }
      if (p.S == 1) {
        if (prow < P) {
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = acc[c + u];
            write8(prow, c, v);
          }
        }
      } else {
        // the operand stages are free: every MMA has completed and every load was consumed
        store_partial_row(ptx::smem_u32(as), q * 32 + lane, acc, p.rpad);
      }
    }
  }
  if (p.S > 1) {
    ptx::cluster_sync();
    if (warp >= 2 && *abort_flag == 0)
      cluster_sum(ptx::smem_u32(as), p.rpad, p.S, split, min(BM, P - p0), threadIdx.x - 64,
                  [&](int lr, int c, const float (&v)[8]) { write8(p0 + lr, c, v); });
    ptx::cluster_sync();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace qlora
