// Expert-parallel row exchange over peer memory.
//
// "Mixture-of-Experts : routage et capacité" slides, "L'idée — Communication" and "Support
// visuel — Communication": a token's row travels to the device that owns its expert, and the
// expert's output travels back.  Instead of posting messages, the rank that holds the rows
// writes them straight into the destination's buffer: each destination buffer is reached
// through a pointer (another process's allocation mapped with CUDA IPC, reached over NVLink
// on a multi-GPU node, or a local buffer), and one launch copies every run of rows.
// Ordering against the destination's own kernels is the caller's (a stream-ordered barrier
// before the copies, so the destination is done with the buffer's previous contents, and one
// after, so its next kernels see the rows).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// One block per row (grid-stride): the row's run by binary search over the runs' row prefix,
// then 16-byte vectors from the source row to the destination row.  A run whose buffer index
// or rows fall outside the given bounds is skipped and reported as invalid input.
__global__ void __launch_bounds__(128) copy_runs_kernel(
    const uint4* __restrict__ src, int64_t src_rows, const unsigned long long* __restrict__ dst_base,
    const int64_t* __restrict__ dst_rows, int n_bufs, const int4* __restrict__ runs,
    const int32_t* __restrict__ run_start, int n_runs, int64_t total_rows, int row_vecs,
    int* status) {
  pdl_wait();
  for (int64_t row = blockIdx.x; row < total_rows; row += gridDim.x) {
    int lo = 0, hi = n_runs;  // largest r with run_start[r] <= row
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (run_start[mid] <= row) lo = mid; else hi = mid;
    }
    const int4 run = runs[lo];  // (src_row, dst_buf, dst_row, rows)
    const int64_t i = row - run_start[lo];
    const int64_t s = (int64_t)run.x + i, d = (int64_t)run.z + i;
    const int b = run.y;
    if (b < 0 || b >= n_bufs || i >= run.w || s < 0 || s >= src_rows || d < 0 ||
        d >= dst_rows[b]) {
      if (threadIdx.x == 0 && status != nullptr) report_status(status, kStatusInvalidInput);
      continue;
    }
    const uint4* sp = src + s * row_vecs;
    uint4* dp = reinterpret_cast<uint4*>(dst_base[b]) + d * row_vecs;
    for (int v = threadIdx.x; v < row_vecs; v += blockDim.x) dp[v] = sp[v];
  }
  // the rows are written before the stream-ordered barrier that follows this kernel
  __threadfence_system();
}

}  // namespace

cudaError_t launch_copy_runs(const void* src, int64_t src_rows, const unsigned long long* dst_base,
                             const int64_t* dst_rows, int n_bufs, const int32_t* runs,
                             const int32_t* run_start, int n_runs, int64_t total_rows,
                             int row_bytes, int* status, cudaStream_t stream, int* launches) {
  if (total_rows <= 0 || n_runs <= 0) return cudaSuccess;
  ++*launches;
  const int64_t grid = std::min<int64_t>(total_rows, (int64_t)tc::num_sms() * 16);
  launch_pdl(copy_runs_kernel, (unsigned)grid, 128, 0, stream, (const uint4*)src, src_rows,
             dst_base, dst_rows, n_bufs, (const int4*)runs, run_start, n_runs, total_rows,
             row_bytes / 16, status);
  return cudaGetLastError();
}

// The allocation that contains a device pointer (CUDA IPC hands out whole allocations, while
// a caching allocator returns pointers inside them).
cudaError_t allocation_base(const void* ptr, void** base) {
  static PFN_cuMemGetAddressRange_v3020 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return cudaErrorNotSupported;
    fn = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(p);
  }
  CUdeviceptr b = 0;
  size_t size = 0;
  if (fn(&b, &size, (CUdeviceptr)ptr) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  *base = reinterpret_cast<void*>(b);
  return cudaSuccess;
}

}  // namespace moe
