// misc_kernels.cu -- small helpers of the step: gathering each slot's current
// set into the caller's contiguous [B][Hs][k] layout, and checking inherited
// sets handed in by the caller.
#include <cuda_runtime.h>
#include <stdint.h>

#include "lyc_plan.h"

namespace lyc {

__global__ void copy_sets_kernel(const CopySetsParams p) {
  const int set = blockIdx.x;
  const int32_t* src = p.src[set];
  int32_t* dst = p.dst + static_cast<int64_t>(set) * p.k;
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
    if (j < p.k_eff) {
      bad |= (v < 0 || v >= p.n);
      if (j > 0) bad |= (v <= s[j - 1]);
    } else {
      bad |= (v != -1);
    }
  }
  if (bad) atomicOr(p.status, kStatusBadIndex);
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
