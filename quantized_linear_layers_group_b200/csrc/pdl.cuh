// pdl.cuh -- programmatic dependent launch (PDL) controls shared by the
// quantise and GEMM kernels.  A kernel launched with the programmatic stream
// serialization attribute may start while the previous kernel in the stream
// is still running; it must call pdl_wait() before reading anything that
// kernel wrote (or writing anything it reads).
#pragma once

namespace qlin {

// Wait until the grids this one depends on have completed and their writes
// are visible (returns at once when the kernel was not launched as a dependent).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Let the next grid in the stream be scheduled now (it still waits in pdl_wait).
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace qlin
