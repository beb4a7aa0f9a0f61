// misc_kernels.cu -- small helpers of the step: gathering each slot's current
// set into the caller's contiguous [B][Hs][k] layout, and checking inherited
// sets handed in by the caller, and writing the current token's K/V rows.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lyc_plan.h"

namespace lyc {

__global__ void copy_sets_kernel(const CopySetsParams p) {
  const int set = blockIdx.x;
  const int32_t* src = p.src[set];
  int32_t* dst = p.dsts ? p.dsts[set] : p.dst + static_cast<int64_t>(set) * p.k;
  for (int j = threadIdx.x; j < p.k; j += blockDim.x) dst[j] = src[j];
  // the step's last launch (every launch of the step has completed before it
  // starts, and the next step's launches start after it ends): the next
  // step's ready flags are told apart from this step's by the epoch
  if (p.epoch && set == 0) {
    const uint32_t e = *p.epoch;
    if (p.pool_cursors)
      for (int j = threadIdx.x; j < p.pool_stride; j += blockDim.x)
        p.pool_cursors[static_cast<int64_t>((e + 1u) & 1u) * p.pool_stride + j] = 0;
    __syncthreads();
    if (threadIdx.x == 0) *p.epoch = e + 1u;
  }
}

__global__ void validate_sets_kernel(const ValidateSetsParams p) {
  const int set = blockIdx.x;
  const int32_t* s = p.sets + static_cast<int64_t>(set) * p.stride;
  bool bad = false;
  for (int j = threadIdx.x; j < p.k; j += blockDim.x) {
    const int32_t v = s[j];
    if (j < p.min_valid) {
      bad |= (v < 0 || v >= p.n);
      if (j > 0) bad |= (v <= s[j - 1]);
    } else if (j < p.k_eff) {
      // a shorter set: valid ascending entries, then only -1
      if (v == -1) {
        bad |= (j + 1 < p.k && s[j + 1] != -1);
      } else {
        bad |= (v < 0 || v >= p.n);
        if (j > 0) bad |= (v <= s[j - 1]);
      }
    } else {
      bad |= (v != -1);
    }
  }
  if (bad) atomicOr(p.status, kStatusBadIndex);
}

// One block per (l, b, g): 16-byte chunks of the K row, then of the V row.
__global__ void append_rows_kernel(const AppendParams p) {
  const int lbg = blockIdx.x;
  const int g = lbg % p.Hkv;
  const int b = (lbg / p.Hkv) % p.B;
  const int l = lbg / (p.Hkv * p.B);
  const int64_t i = p.n[b] - 1;
  int64_t off = static_cast<int64_t>(l) * p.s_layer + static_cast<int64_t>(g) * p.s_head;
  if (p.bt)
    off += static_cast<int64_t>(p.bt[static_cast<int64_t>(b) * p.max_blocks + i / p.page_rows]) * p.s_page +
           (i % p.page_rows) * p.s_token;
  else
    off += static_cast<int64_t>(b) * p.s_batch + i * p.s_token;
  const int64_t dst = off * p.elem_bytes;
  const int64_t src = static_cast<int64_t>(lbg) * p.row_bytes;
  const int chunks = p.row_bytes / 16;
  for (int c = threadIdx.x; c < 2 * chunks; c += blockDim.x) {
    const bool isv = c >= chunks;
    const int cc = isv ? c - chunks : c;
    const uint4 x = *reinterpret_cast<const uint4*>((isv ? p.v_new : p.k_new) + src + 16 * cc);
    *reinterpret_cast<uint4*>((isv ? p.v : p.k) + dst + 16 * cc) = x;
  }
}

cudaError_t append_rows_launch(const AppendParams* p, cudaStream_t stream) {
  const int blocks = p->L * p->B * p->Hkv;
  if (blocks <= 0) return cudaSuccess;
  append_rows_kernel<<<blocks, 64, 0, stream>>>(*p);
  return cudaGetLastError();
}

cudaError_t copy_sets_launch(const CopySetsParams* p, cudaStream_t stream) {
  if (p->nsets <= 0) return cudaSuccess;  // never the case: a step has B * Hs >= 1 sets
  copy_sets_kernel<<<p->nsets, 256, 0, stream>>>(*p);
  return cudaGetLastError();
}

cudaError_t validate_sets_launch(const ValidateSetsParams* p, cudaStream_t stream) {
  if (p->nsets <= 0) return cudaSuccess;
  validate_sets_kernel<<<p->nsets, 256, 0, stream>>>(*p);
  return cudaGetLastError();
}

}  // namespace lyc
