// Device-side helpers shared by the kernels of the MoE layer (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device status codes (same values as moe_status in include/moe.h).
enum : int { kStatusOk = 0, kStatusInvalidInput = 4, kStatusTimeout = 5 };

// Record a device-side finding: the first error since the last host check wins.
__device__ __forceinline__ void report_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Token-tile size of the dispatch kernels (tokens ranked by one warp in order).
constexpr int kRankTile = 32;

// Programmatic dependent launch.  Every kernel of the library is launched with programmatic
// stream serialisation (launch_pdl), so the GPU may schedule it while its predecessor on the
// stream is still running; pdl_wait() returns once that predecessor has completed and its
// memory is visible, and every kernel calls it before touching global memory.  The chain
// stays transitive because each kernel waits before it finishes.  pdl_release() lets the
// successor be scheduled before this grid ends (the persistent GEMMs call it once their
// last loads are issued); without it the successor is released at exit.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace moe
