// qlora_groups.cuh -- device-side tile tables for grouped (mixture-of-experts) launches.
//
// Expert e owns rows [off[e], off[e+1]) of the expert-packed activations ("Quantized weights,
// full precision: The math behind 75% cheaper fine-tuning", "LoRA operations and quantization":
// LoRA on the mxfp4 experts of an MoE model).  The offsets live in device memory, so every CTA
// builds the same small table in shared memory at start-up: per expert its row range and the
// index of its first tile, where an expert with c rows has ceil(c / rows_per_tile) row tiles,
// each repeated `per_row_tile` times (column tiles or contraction splits).  A single layer is the
// same table with one expert covering rows [0, M).
#pragma once
#include <cstdint>

namespace qlora {

constexpr int kMaxExperts = 1024;

struct GroupView {
  const int* off;     // shared: [E+1] row offsets
  const int* first;   // shared: [E+1] first tile of each expert; first[E] = total tiles
  int E;
  __device__ __forceinline__ int total() const { return first[E]; }
  // expert owning tile t (0 <= t < total): the last e with first[e] <= t
  __device__ __forceinline__ int expert_of(int t) const {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (first[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
};

// Build the table (call from all threads of the CTA; ends with __syncthreads()).  g_off == nullptr
// means one expert of M rows.  Invalid offsets (off[0] != 0, decreasing, or off[E] != M) record
// QLORA_ERR_INVALID_ARG in *status and give an empty table.
__device__ __forceinline__ GroupView build_group_view(const int32_t* g_off, int E, int M,
                                                      int rows_per_tile, int per_row_tile,
                                                      int* s_off, int* s_first, int* status) {
  if (g_off == nullptr) E = 1;
  for (int e = threadIdx.x; e <= E; e += blockDim.x)
    s_off[e] = g_off ? g_off[e] : (e == 0 ? 0 : M);
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = s_off[0] == 0 && s_off[E] == M;
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      const int c = s_off[e + 1] - s_off[e];
      if (c < 0) ok = false;
      s_first[e] = acc;
      acc += (c > 0 ? (c + rows_per_tile - 1) / rows_per_tile : 0) * per_row_tile;
    }
    s_first[E] = ok ? acc : 0;
    if (!ok) {
      for (int e = 0; e < E; ++e) s_first[e] = 0;
      if (status) atomicCAS(status, 0, 1 /* QLORA_ERR_INVALID_ARG */);
    }
  }
  __syncthreads();
  return GroupView{s_off, s_first, E};
}

}  // namespace qlora
