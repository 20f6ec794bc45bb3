// nomas_selftest_bounded_wait: a bounded wait that is made to run out, on the device.
//
// Every kernel of this library waits on mbarriers with mbar_wait, which gives
// up after NOMAS_WAIT_NS of device time, records NOMAS_DEVERR_TIMEOUT in the
// workspace status word and raises the CTA's abort flag so that the other
// roles of the CTA stop waiting too. This self-test runs that code path for
// real: one CTA waits on an mbarrier that nothing ever arrives on (no fault,
// trap or endless loop is involved), and a second warp waits on another such
// barrier until it sees the abort flag. The host reads the outcome through
// nomas_device_status, and the context stays usable afterwards.
#include "nomas_div127.cuh"
#include "nomas_internal.h"
#include "nomas_ptx.cuh"

namespace nomas {
namespace {

__global__ void __launch_bounds__(64, 1) selftest_wait_kernel(unsigned* status) {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_flag;
    const uint32_t b0 = smem_u32(&bars[0]), b1 = smem_u32(&bars[1]);
    if (threadIdx.x == 0) {
        mbar_init(b0, 1);
        mbar_init(b1, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const WaitCtl ctl{&abort_flag, status};
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0 && lane == 0) {
        // runs out after NOMAS_WAIT_NS: sets the status bit and the abort flag
        if (!mbar_wait(b0, 0, ctl)) status[1] = 1u;
    } else if (warp == 1 && lane == 0) {
        // the second role learns of the abort through the flag and returns false
        if (!mbar_wait(b1, 0, ctl)) status[2] = 1u;
    }
}

// Every non-negative fp32 bit pattern x in [0, 2^31): div127_rn(x) against the
// IEEE quotient __fdiv_rn(x, 127). A mismatch is counted when the bit
// patterns differ, unless both results are NaN. out[0] counts mismatches,
// out[1] keeps the smallest mismatching input pattern (0xFFFFFFFF if none).
__global__ void __launch_bounds__(256) selftest_div127_kernel(unsigned* out) {
    unsigned local = 0, first = 0xFFFFFFFFu;
    const unsigned stride = gridDim.x * blockDim.x;
    for (unsigned u = blockIdx.x * blockDim.x + threadIdx.x; u < 0x80000000u; u += stride) {
        const float x = __uint_as_float(u);
        const float a = div127_rn(x), b = __fdiv_rn(x, 127.0f);
        const bool same = __float_as_uint(a) == __float_as_uint(b) || (a != a && b != b);
        if (!same) {
            ++local;
            first = min(first, u);
        }
    }
    for (int off = 16; off >= 1; off >>= 1) {
        local += __shfl_xor_sync(0xFFFFFFFFu, local, off);
        first = min(first, __shfl_xor_sync(0xFFFFFFFFu, first, off));
    }
    if ((threadIdx.x & 31) == 0 && local) {
        atomicAdd(&out[0], local);
        atomicMin(&out[1], first);
    }
}

} // namespace
} // namespace nomas

extern "C" int nomas_selftest_bounded_wait(void* workspace, void* stream) {
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 15u)) return NOMAS_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(static_cast<unsigned*>(workspace) + 1, 0, 2 * sizeof(unsigned), s) != cudaSuccess)
        return NOMAS_ERR_CUDA;
    nomas::selftest_wait_kernel<<<1, 64, 0, s>>>(static_cast<unsigned*>(workspace));
    return cudaGetLastError() == cudaSuccess ? NOMAS_OK : NOMAS_ERR_CUDA;
}

extern "C" int nomas_selftest_div127(void* result, void* stream) {
    if (!result || (reinterpret_cast<uintptr_t>(result) & 7u)) return NOMAS_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned* r = static_cast<unsigned*>(result);
    if (cudaMemsetAsync(r, 0, sizeof(unsigned), s) != cudaSuccess ||
        cudaMemsetAsync(r + 1, 0xFF, sizeof(unsigned), s) != cudaSuccess)
        return NOMAS_ERR_CUDA;
    // 148 SMs x 8 blocks of 256 threads: each thread checks 7,085 inputs
    nomas::selftest_div127_kernel<<<148 * 8, 256, 0, s>>>(r);
    return cudaGetLastError() == cudaSuccess ? NOMAS_OK : NOMAS_ERR_CUDA;
}
