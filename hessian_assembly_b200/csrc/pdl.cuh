// pdl.cuh -- programmatic dependent launch between the kernels of one step.
//
// A kernel launched with programmatic stream serialization may start before
// the previous kernel on its stream has finished: its blocks are scheduled
// once every block of the previous kernel has signalled (or exited), load
// what does not depend on that kernel, and wait before reading its results.
// The launch latency and ramp of a dependent kernel then overlap the tail of
// its predecessor.
//
// Use it only for a kernel that reads (a) what its immediate predecessor
// wrote, after grid_dependency_wait(), and (b) data written by work that had
// finished before that predecessor started, i.e. a predecessor launched the
// ordinary way.  After the wait, writes of a grid two steps back in a chain
// of such launches were not visible: in a chain of five the third kernel
// read stale row offsets from the first.  So every use here is one ordinary
// launch followed by one programmatic launch.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace mad {

// Wait until the previous kernel on the stream has finished and its writes
// are visible (returns at once for a kernel launched the ordinary way).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Let the next kernel on the stream start (it still waits for the results).
__device__ __forceinline__ void grid_dependents_may_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches k<<<grid, block, smem, s>>>(args...) with programmatic stream
// serialization allowed, when s is not being captured into a CUDA graph.
// Under capture the kernel is launched the ordinary way (a full dependency
// on the previous node): the overlap is only taken where the stream itself
// orders the kernels.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = cs == cudaStreamCaptureStatusNone ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

}  // namespace mad
