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

// One warp ranks the assignments of `ntok` consecutive tokens in token order, continuing the
// per-expert counters cnt[] (shared memory): sid[t * k + j] is the expert of slot j of token
// t, or -1 for none.  rank(t, e) = the number of earlier tokens that chose e.  An expert listed
// twice by one token keeps its first slot only.  out(t, j, r) receives each slot's rank (-1 for
// none); returns true (in every lane) if some token listed an expert twice.
template <typename Out>
__device__ __forceinline__ bool warp_rank_walk(const int32_t* sid, int ntok, int k,
                                               int32_t* cnt, int lane, Out&& out) {
  bool bad = false;
  for (int t = 0; t < ntok; ++t) {
    int v = lane < k ? sid[t * k + lane] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, v);
    if (v >= 0 && (__ffs(peers) - 1) != lane) {
      bad = true;
      v = -1;
    }
    int r = -1;
    if (v >= 0) {
      r = cnt[v];
      cnt[v] = r + 1;
    }
    if (lane < k) out(t, lane, r);
    __syncwarp();
  }
  return __any_sync(0xffffffffu, bad);
}

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
