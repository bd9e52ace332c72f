// k_tc.cu -- tensor-core (tcgen05 + TMA) reduce and apply kernels for bf16.
#include <cuda_runtime.h>

#include "la_internal.cuh"

namespace la {

// Raised by a bounded device-side wait that gave up.
__device__ unsigned int g_wait_flag = 0;

bool tc_available() { return false; }

int launch_reduce_tc(const void *, const void *, float *, const Plan &, cudaStream_t) { return -1; }

int launch_apply_tc(const void *, void *, const void *, const Plan &, cudaStream_t) { return -1; }

int read_and_clear_device_flag(cudaStream_t s, unsigned *flag_out) {
    unsigned zero = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(flag_out, g_wait_flag, sizeof(unsigned)) != cudaSuccess) return -1;
    if (*flag_out && cudaMemcpyToSymbol(g_wait_flag, &zero, sizeof(unsigned)) != cudaSuccess) return -1;
    return 0;
}

}  // namespace la
