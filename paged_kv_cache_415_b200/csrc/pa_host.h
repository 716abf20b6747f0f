// pa_host.h -- host-side argument checks shared by the C-ABI entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "pa.h"

namespace pa {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
inline bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

inline bool supported_head_dim(int32_t d) { return d == 64 || d == 128; }
inline bool supported_block_size(int32_t b) { return b == 8 || b == 16 || b == 32; }
inline bool supported_dtype(int32_t t) { return t == PA_DTYPE_F16 || t == PA_DTYPE_BF16; }
// One-byte pool element types (block copies and swaps move them as bytes).
inline bool code_dtype(int32_t t) { return t == PA_DTYPE_FP8_E4M3 || t == PA_DTYPE_INT8; }

// Launch-error check after a kernel launch.
inline pa_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Launch with programmatic stream serialisation: the kernel may begin while
// the previous kernel in the stream finishes; every kernel of this library
// waits (griddepcontrol.wait) before touching global memory, so only the
// launch and ramp-up overlap.
template <typename... KArgs, typename... Args>
inline pa_status launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t stream, Args&&... args)
{
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
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess
               ? launch_status()
               : PA_ERR_CUDA;
}

}  // namespace pa
