// Copies of a decode step's inputs and output between host memory the device
// can read and write (page-locked, mapped) and device memory, as one small
// kernel instead of DMA copies: the step of socket_decode_step_host.
#pragma once

#include <cstddef>
#include <cstdint>

#include "common.cuh"

namespace hst {

// Up to three strided row copies in one launch: job j copies rows[j] rows of
// row16[j] 16-byte words from src[j] (pitch src_pitch[j] bytes) to dst[j]
// (pitch dst_pitch[j] bytes). Every address and pitch is a multiple of 16
// bytes. Plain 16-byte loads and stores, one word per thread and step.
struct StepCopyParams {
  const char* src[3];
  char* dst[3];
  size_t src_pitch[3], dst_pitch[3];
  int rows[3], row16[3];
  int jobs;
};

constexpr int STEP_COPY_THREADS = 256;

__global__ void __launch_bounds__(STEP_COPY_THREADS) step_copy_kernel(const StepCopyParams p) {
  // launched as the programmatic dependent of the kernel that writes its
  // source, it reads only after that kernel completed (a no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int j = 0; j < p.jobs; ++j) {
    const long long words = (long long)p.rows[j] * p.row16[j];
    for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < words;
         w += (long long)gridDim.x * blockDim.x) {
      const long long r = w / p.row16[j], c = w % p.row16[j];
      const uint4 v = *reinterpret_cast<const uint4*>(p.src[j] + r * (long long)p.src_pitch[j] + 16 * c);
      *reinterpret_cast<uint4*>(p.dst[j] + r * (long long)p.dst_pitch[j] + 16 * c) = v;
    }
  }
}

}  // namespace hst
