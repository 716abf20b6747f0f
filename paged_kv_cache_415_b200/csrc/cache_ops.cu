// cache_ops.cu -- the two kernels that feed the paged KV cache:
//   reshape_and_cache : scatter this step's new K/V rows into their slots
//   copy_blocks       : copy-on-write block copies
//
// Both are bit copies moved in 16-byte vectors; neither looks at values,
// so one instance serves fp16 and bf16.
//
// Pages cited (title, then section):
//   [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
//   [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
//   [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "pa.h"
#include "pa_codes.cuh"
#include "pa_common.cuh"
#include "pa_host.h"

namespace pa {

constexpr int kCopyThreads = 256;
constexpr int kCopyVecsPerThread = 4;

// Grid (token, chunk of the row).  The pools are [num_slots][Hkv][D], so a
// token's K row (all kv heads) is one contiguous run of row_vecs 16-byte
// vectors at slot * row_vecs ([Practice §3.3 按需分配策略], step 4: write the
// new token's KV vectors into the slot the allocator gave it).  Each thread
// moves up to kCacheVecsPerThread vectors of K and of V, all loads first.
constexpr int kCacheThreads = 128;
constexpr int kCacheVecsPerThread = 2;

__global__ void __launch_bounds__(kCacheThreads) reshape_and_cache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int32_t row_vecs,
    int64_t num_slots, int32_t* d_status)
{
    grid_dependency_wait();
    allow_dependents();
    const int64_t t = blockIdx.x;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;                       // padding token
    if (slot >= num_slots) {
        if (threadIdx.x == 0 && blockIdx.y == 0) status_or(d_status, PA_STATUS_BAD_SLOT);
        return;
    }
    const uint4* ks = key + t * row_vecs;
    const uint4* vs = value + t * row_vecs;
    uint4* kd = k_cache + slot * row_vecs;
    uint4* vd = v_cache + slot * row_vecs;
    const int32_t base = blockIdx.y * kCacheThreads * kCacheVecsPerThread + threadIdx.x;
    uint4 a[kCacheVecsPerThread], b[kCacheVecsPerThread];
#pragma unroll
    for (int j = 0; j < kCacheVecsPerThread; ++j) {
        const int32_t i = base + j * kCacheThreads;
        if (i < row_vecs) {
            a[j] = ld_nc_v4(ks + i);
            b[j] = ld_nc_v4(vs + i);
        }
    }
#pragma unroll
    for (int j = 0; j < kCacheVecsPerThread; ++j) {
        const int32_t i = base + j * kCacheThreads;
        if (i < row_vecs) {
            kd[i] = a[j];
            vd[i] = b[j];
        }
    }
}

// Quantising variant for one-byte pools (e4m3 or int8, pa_codes.cuh): each
// vector of 8 input elements becomes 8 codes of fp32(x) * inv_scale.
template <typename Codes, typename T>
__global__ void __launch_bounds__(kCacheThreads) reshape_and_cache_q8_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint2* __restrict__ k_cache,
    uint2* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int32_t row_vecs,
    int64_t num_slots, float k_inv, float v_inv, int32_t* d_status)
{
    grid_dependency_wait();
    allow_dependents();
    const int64_t t = blockIdx.x;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (threadIdx.x == 0 && blockIdx.y == 0) status_or(d_status, PA_STATUS_BAD_SLOT);
        return;
    }
    const int32_t base = blockIdx.y * kCacheThreads * kCacheVecsPerThread + threadIdx.x;
    uint4 a[kCacheVecsPerThread], b[kCacheVecsPerThread];
#pragma unroll
    for (int j = 0; j < kCacheVecsPerThread; ++j) {
        const int32_t i = base + j * kCacheThreads;
        if (i < row_vecs) {
            a[j] = ld_nc_v4(key + t * row_vecs + i);
            b[j] = ld_nc_v4(value + t * row_vecs + i);
        }
    }
#pragma unroll
    for (int j = 0; j < kCacheVecsPerThread; ++j) {
        const int32_t i = base + j * kCacheThreads;
        if (i < row_vecs) {
            k_cache[slot * row_vecs + i] = encode8<Codes, T>(a[j], k_inv);
            v_cache[slot * row_vecs + i] = encode8<Codes, T>(b[j], v_inv);
        }
    }
}

// Row-scaled variant: one warp per (token, kv head) quantises that row of K
// and of V with a scale of its own (quantise_row_warp: s = max|x| / kMax,
// codes of x * (1 / s)) and stores the codes at the slot and the scales at
// [slot / B][kv head][slot % B] of the scale pools.  Grid (token, group of
// four kv heads).
constexpr int kRowWarps = kCacheThreads / 32;

template <typename Codes, typename T, int D>
__global__ void __launch_bounds__(kCacheThreads) reshape_and_cache_rowscale_kernel(
    const T* __restrict__ key, const T* __restrict__ value, uint8_t* __restrict__ k_cache,
    uint8_t* __restrict__ v_cache, float* __restrict__ k_scales, float* __restrict__ v_scales,
    const int64_t* __restrict__ slot_mapping, int32_t num_kv_heads, int32_t block_size,
    int64_t num_slots, int32_t* d_status)
{
    grid_dependency_wait();
    allow_dependents();
    const int64_t t = blockIdx.x;
    const int g = blockIdx.y * kRowWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;                       // padding token
    if (slot >= num_slots) {
        if (threadIdx.x == 0 && blockIdx.y == 0) status_or(d_status, PA_STATUS_BAD_SLOT);
        return;
    }
    if (g >= num_kv_heads) return;              // warp-uniform
    const int64_t src = (t * num_kv_heads + g) * D;
    const int64_t dst = (slot * num_kv_heads + g) * D;
    const int64_t si = ((slot / block_size) * num_kv_heads + g) * block_size + slot % block_size;
    uint4 kx = make_uint4(0, 0, 0, 0), vx = make_uint4(0, 0, 0, 0);
    if (lane < D / 8) {
        kx = ld_nc_v4(key + src + lane * 8);
        vx = ld_nc_v4(value + src + lane * 8);
    }
    float ks, vs;
    const uint2 kc = quantise_row_warp<Codes, T, D>(kx, ks);
    const uint2 vc = quantise_row_warp<Codes, T, D>(vx, vs);
    if (lane < D / 8) {
        *reinterpret_cast<uint2*>(k_cache + dst + lane * 8) = kc;
        *reinterpret_cast<uint2*>(v_cache + dst + lane * 8) = vc;
    }
    if (lane == 0) {
        k_scales[si] = ks;
        v_scales[si] = vs;
    }
}

// Grid (pair, K-or-V, chunk of the block).  Whole-block bit copy src -> dst
// ([VM-paging, 写时复制与块共享机制]; [Practice §4.1 共享内存管理] step 2).
// The first CTA of each pair also checks the pair against all the others:
// a destination that appears twice, or that another pair reads, makes the
// result order-dependent, which is flagged.
__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(
    uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
    const int64_t* __restrict__ block_mapping, int32_t num_pairs, int64_t block_vecs,
    int64_t num_blocks, int32_t* d_status)
{
    grid_dependency_wait();
    allow_dependents();
    const int32_t pair = blockIdx.x;
    const int64_t src = block_mapping[2 * pair];
    const int64_t dst = block_mapping[2 * pair + 1];
    const bool first_cta = blockIdx.y == 0 && blockIdx.z == 0;
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (first_cta && threadIdx.x == 0) status_or(d_status, PA_STATUS_BAD_BLOCK);
        return;
    }
    if (first_cta && d_status != nullptr) {
        bool conflict = false;
        for (int32_t j = threadIdx.x; j < num_pairs; j += blockDim.x) {
            if (j == pair) continue;
            const int64_t sj = block_mapping[2 * j], dj = block_mapping[2 * j + 1];
            if (dj == dst && j < pair) conflict = true;
            if (sj == dst && sj != dj) conflict = true;
        }
        if (__syncthreads_or(conflict) && threadIdx.x == 0) status_or(d_status, PA_STATUS_COPY_CONFLICT);
    }
    if (src == dst) return;
    uint4* base = blockIdx.y == 0 ? k_cache : v_cache;
    const uint4* s = base + src * block_vecs;
    uint4* d = base + dst * block_vecs;
    const int64_t begin = static_cast<int64_t>(blockIdx.z) * kCopyThreads * kCopyVecsPerThread;
    const int64_t end = min(block_vecs, begin + static_cast<int64_t>(kCopyThreads) * kCopyVecsPerThread);
    uint4 buf[kCopyVecsPerThread];
#pragma unroll
    for (int k = 0; k < kCopyVecsPerThread; ++k) {
        const int64_t i = begin + threadIdx.x + static_cast<int64_t>(k) * kCopyThreads;
        if (i < end) buf[k] = s[i];
    }
#pragma unroll
    for (int k = 0; k < kCopyVecsPerThread; ++k) {
        const int64_t i = begin + threadIdx.x + static_cast<int64_t>(k) * kCopyThreads;
        if (i < end) d[i] = buf[k];
    }
}

// Grid (pair, K-or-V, chunk of the block).  Whole-block bit copy from one
// pool to another, either of which may be pinned host memory reached over
// the host link ([VM-paging, 显存管理与调度策略设计], eviction to CPU memory and
// back).  Every thread keeps kSwapVecsPerThread 16-byte loads in flight, so
// the link's read latency is covered.  The first CTA of each pair checks
// the pair against the others (repeated destinations; with one shared pool,
// also destinations that other pairs read).
constexpr int kSwapThreads = 256;
constexpr int kSwapVecsPerThread = 8;

__global__ void __launch_bounds__(kSwapThreads) swap_blocks_kernel(
    const uint4* __restrict__ src_k, const uint4* __restrict__ src_v, uint4* __restrict__ dst_k,
    uint4* __restrict__ dst_v, const int64_t* __restrict__ block_mapping, int32_t num_pairs,
    int64_t block_vecs, int64_t src_num_blocks, int64_t dst_num_blocks, int32_t same_pool,
    int32_t* d_status)
{
    grid_dependency_wait();
    allow_dependents();
    const int32_t pair = blockIdx.x;
    const int64_t src = block_mapping[2 * pair];
    const int64_t dst = block_mapping[2 * pair + 1];
    const bool first_cta = blockIdx.y == 0 && blockIdx.z == 0;
    if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
        if (first_cta && threadIdx.x == 0) status_or(d_status, PA_STATUS_BAD_BLOCK);
        return;
    }
    if (first_cta && d_status != nullptr) {
        bool conflict = false;
        for (int32_t j = threadIdx.x; j < num_pairs; j += blockDim.x) {
            if (j == pair) continue;
            const int64_t sj = block_mapping[2 * j], dj = block_mapping[2 * j + 1];
            if (dj == dst && j < pair) conflict = true;
            if (same_pool && sj == dst && sj != dj) conflict = true;
        }
        if (__syncthreads_or(conflict) && threadIdx.x == 0) status_or(d_status, PA_STATUS_COPY_CONFLICT);
    }
    if (same_pool && src == dst) return;
    const uint4* s = (blockIdx.y == 0 ? src_k : src_v) + src * block_vecs;
    uint4* d = (blockIdx.y == 0 ? dst_k : dst_v) + dst * block_vecs;
    const int64_t begin = static_cast<int64_t>(blockIdx.z) * kSwapThreads * kSwapVecsPerThread;
    const int64_t end = min(block_vecs, begin + static_cast<int64_t>(kSwapThreads) * kSwapVecsPerThread);
    uint4 buf[kSwapVecsPerThread];
#pragma unroll
    for (int k = 0; k < kSwapVecsPerThread; ++k) {
        const int64_t i = begin + threadIdx.x + static_cast<int64_t>(k) * kSwapThreads;
        if (i < end) buf[k] = s[i];
    }
#pragma unroll
    for (int k = 0; k < kSwapVecsPerThread; ++k) {
        const int64_t i = begin + threadIdx.x + static_cast<int64_t>(k) * kSwapThreads;
        if (i < end) d[i] = buf[k];
    }
}

// Pools the calls accept: 16-bit pools (head_dim 64 or 128); with
// allow_codes also one-byte code pools, and row-scale pools (PA_DTYPE_F32,
// head_dim 1: a block holds block_size x num_kv_heads fp32 scales).
static pa_status check_pool_shape(int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  int64_t num_blocks, int32_t dtype, bool allow_codes = false)
{
    if (num_kv_heads <= 0 || num_blocks <= 0 || head_dim <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (allow_codes && dtype == PA_DTYPE_F32)
        return head_dim == 1 && supported_block_size(block_size) ? PA_OK : PA_ERR_UNSUPPORTED;
    const bool dtype_ok = supported_dtype(dtype) || (allow_codes && code_dtype(dtype));
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size) || !dtype_ok)
        return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

// Bytes of one element of a pool of this type.
static int pool_elem_bytes(int32_t dtype)
{
    return dtype == PA_DTYPE_F32 ? 4 : code_dtype(dtype) ? 1 : 2;
}

}  // namespace pa

extern "C" pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                          void* v_cache, const int64_t* slot_mapping,
                                          int32_t num_tokens, int32_t num_kv_heads,
                                          int32_t head_dim, int32_t block_size,
                                          int64_t num_blocks, pa_dtype dtype, int32_t* d_status,
                                          pa_stream_t stream)
{
    using namespace pa;
    if (num_tokens < 0) return PA_ERR_INVALID_ARG;
    pa_status st = check_pool_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (st != PA_OK) return st;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned8(slot_mapping) || (d_status && !aligned4(d_status)))
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    const int32_t row_vecs = num_kv_heads * head_dim * 2 / 16;
    const int32_t per_cta = kCacheThreads * kCacheVecsPerThread;
    const int32_t chunks = (row_vecs + per_cta - 1) / per_cta;
    if (chunks > 65535) return PA_ERR_UNSUPPORTED;
    dim3 grid(num_tokens, chunks);
    return launch_overlapped(reshape_and_cache_kernel, grid, dim3(kCacheThreads), 0, stream,
                             static_cast<const uint4*>(key), static_cast<const uint4*>(value),
                             static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                             slot_mapping, row_vecs, num_blocks * block_size, d_status);
}

extern "C" pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                                    int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t block_size, int64_t num_blocks, pa_dtype dtype,
                                    int32_t* d_status, pa_stream_t stream)
{
    using namespace pa;
    if (num_pairs < 0) return PA_ERR_INVALID_ARG;
    pa_status st = check_pool_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype, true);
    if (st != PA_OK) return st;
    if (!k_cache || !v_cache || !block_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned8(block_mapping) ||
        (d_status && !aligned4(d_status)))
        return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    const int elem_bytes = pool_elem_bytes(dtype);
    const int64_t block_vecs =
        static_cast<int64_t>(block_size) * num_kv_heads * head_dim * elem_bytes / 16;
    const int64_t per_cta = static_cast<int64_t>(kCopyThreads) * kCopyVecsPerThread;
    const int64_t chunks = (block_vecs + per_cta - 1) / per_cta;
    if (chunks > 65535) return PA_ERR_UNSUPPORTED;
    dim3 grid(num_pairs, 2, static_cast<unsigned>(chunks));
    return launch_overlapped(copy_blocks_kernel, grid, dim3(kCopyThreads), 0, stream,
                             static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                             block_mapping, num_pairs, block_vecs, num_blocks, d_status);
}

namespace pa {
template <typename Codes>
static pa_status reshape_and_cache_q8(const void* key, const void* value, void* k_cache,
                                      void* v_cache, const int64_t* slot_mapping,
                                      int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t block_size, int64_t num_blocks, pa_dtype dtype,
                                      float k_scale, float v_scale, int32_t* d_status,
                                      pa_stream_t stream)
{
    if (num_tokens < 0) return PA_ERR_INVALID_ARG;
    pa_status st = check_pool_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (st != PA_OK) return st;
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(k_scale) || !isfinite(v_scale))
        return PA_ERR_INVALID_ARG;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned8(slot_mapping) || (d_status && !aligned4(d_status)))
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    const int32_t row_vecs = num_kv_heads * head_dim / 8;
    const int32_t per_cta = kCacheThreads * kCacheVecsPerThread;
    const int32_t chunks = (row_vecs + per_cta - 1) / per_cta;
    if (chunks > 65535) return PA_ERR_UNSUPPORTED;
    dim3 grid(num_tokens, chunks);
    const float k_inv = 1.0f / k_scale, v_inv = 1.0f / v_scale;
    auto kernel = dtype == PA_DTYPE_F16 ? reshape_and_cache_q8_kernel<Codes, __half>
                                        : reshape_and_cache_q8_kernel<Codes, __nv_bfloat16>;
    return launch_overlapped(kernel, grid, dim3(kCacheThreads), 0, stream,
                             static_cast<const uint4*>(key), static_cast<const uint4*>(value),
                             static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache),
                             slot_mapping, row_vecs, num_blocks * block_size, k_inv, v_inv,
                             d_status);
}
}  // namespace pa

extern "C" pa_status pa_reshape_and_cache_fp8(const void* key, const void* value, void* k_cache,
                                              void* v_cache, const int64_t* slot_mapping,
                                              int32_t num_tokens, int32_t num_kv_heads,
                                              int32_t head_dim, int32_t block_size,
                                              int64_t num_blocks, pa_dtype dtype, float k_scale,
                                              float v_scale, int32_t* d_status,
                                              pa_stream_t stream)
{
    return pa::reshape_and_cache_q8<pa::E4m3Codes>(key, value, k_cache, v_cache, slot_mapping,
                                                   num_tokens, num_kv_heads, head_dim, block_size,
                                                   num_blocks, dtype, k_scale, v_scale, d_status,
                                                   stream);
}

extern "C" pa_status pa_reshape_and_cache_int8(const void* key, const void* value, void* k_cache,
                                               void* v_cache, const int64_t* slot_mapping,
                                               int32_t num_tokens, int32_t num_kv_heads,
                                               int32_t head_dim, int32_t block_size,
                                               int64_t num_blocks, pa_dtype dtype, float k_scale,
                                               float v_scale, int32_t* d_status,
                                               pa_stream_t stream)
{
    return pa::reshape_and_cache_q8<pa::Int8Codes>(key, value, k_cache, v_cache, slot_mapping,
                                                   num_tokens, num_kv_heads, head_dim, block_size,
                                                   num_blocks, dtype, k_scale, v_scale, d_status,
                                                   stream);
}

namespace pa {
template <typename Codes, typename T>
static pa_status launch_rowscale_write(const void* key, const void* value, void* k_cache,
                                       void* v_cache, float* k_scales, float* v_scales,
                                       const int64_t* slot_mapping, dim3 grid, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t block_size, int64_t num_slots,
                                       int32_t* d_status, pa_stream_t stream)
{
    auto kernel = head_dim == 128 ? reshape_and_cache_rowscale_kernel<Codes, T, 128>
                                  : reshape_and_cache_rowscale_kernel<Codes, T, 64>;
    return launch_overlapped(kernel, grid, dim3(kCacheThreads), 0, stream,
                             static_cast<const T*>(key), static_cast<const T*>(value),
                             static_cast<uint8_t*>(k_cache), static_cast<uint8_t*>(v_cache),
                             k_scales, v_scales, slot_mapping, num_kv_heads, block_size, num_slots,
                             d_status);
}

template <typename Codes>
static pa_status reshape_and_cache_rowscale(const void* key, const void* value, void* k_cache,
                                            void* v_cache, float* k_scales, float* v_scales,
                                            const int64_t* slot_mapping, int32_t num_tokens,
                                            int32_t num_kv_heads, int32_t head_dim,
                                            int32_t block_size, int64_t num_blocks, pa_dtype dtype,
                                            int32_t* d_status, pa_stream_t stream)
{
    if (num_tokens < 0) return PA_ERR_INVALID_ARG;
    pa_status st = check_pool_shape(num_kv_heads, head_dim, block_size, num_blocks, dtype);
    if (st != PA_OK) return st;
    if (!key || !value || !k_cache || !v_cache || !k_scales || !v_scales || !slot_mapping)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(k_scales) || !aligned16(v_scales) || !aligned8(slot_mapping) ||
        (d_status && !aligned4(d_status)))
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    const int32_t groups = (num_kv_heads + kRowWarps - 1) / kRowWarps;
    if (groups > 65535) return PA_ERR_UNSUPPORTED;
    dim3 grid(num_tokens, groups);
    const int64_t num_slots = num_blocks * block_size;
    return dtype == PA_DTYPE_F16
               ? launch_rowscale_write<Codes, __half>(key, value, k_cache, v_cache, k_scales,
                                                      v_scales, slot_mapping, grid, num_kv_heads,
                                                      head_dim, block_size, num_slots, d_status,
                                                      stream)
               : launch_rowscale_write<Codes, __nv_bfloat16>(
                     key, value, k_cache, v_cache, k_scales, v_scales, slot_mapping, grid,
                     num_kv_heads, head_dim, block_size, num_slots, d_status, stream);
}
}  // namespace pa

extern "C" pa_status pa_reshape_and_cache_fp8_rowscale(
    const void* key, const void* value, void* k_cache, void* v_cache, float* k_scales,
    float* v_scales, const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int64_t num_blocks, pa_dtype dtype, int32_t* d_status,
    pa_stream_t stream)
{
    return pa::reshape_and_cache_rowscale<pa::E4m3Codes>(
        key, value, k_cache, v_cache, k_scales, v_scales, slot_mapping, num_tokens, num_kv_heads,
        head_dim, block_size, num_blocks, dtype, d_status, stream);
}

extern "C" pa_status pa_reshape_and_cache_int8_rowscale(
    const void* key, const void* value, void* k_cache, void* v_cache, float* k_scales,
    float* v_scales, const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int64_t num_blocks, pa_dtype dtype, int32_t* d_status,
    pa_stream_t stream)
{
    return pa::reshape_and_cache_rowscale<pa::Int8Codes>(
        key, value, k_cache, v_cache, k_scales, v_scales, slot_mapping, num_tokens, num_kv_heads,
        head_dim, block_size, num_blocks, dtype, d_status, stream);
}

namespace pa {
// The address the device uses for p: device and managed memory as is,
// pinned host memory through its mapping; anything else (pageable host
// memory, an unknown pointer) is refused, so no kernel ever dereferences it.
static bool device_address(const void* p, const void** out)
{
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    switch (attr.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
        *out = p;
        return true;
    case cudaMemoryTypeHost:
        if (attr.devicePointer == nullptr) return false;
        *out = attr.devicePointer;
        return true;
    default:
        return false;
    }
}
}  // namespace pa

extern "C" pa_status pa_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                                    const int64_t* block_mapping, int32_t num_pairs,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                    int64_t src_num_blocks, int64_t dst_num_blocks, pa_dtype dtype,
                                    int32_t* d_status, pa_stream_t stream)
{
    using namespace pa;
    if (num_pairs < 0 || dst_num_blocks <= 0) return PA_ERR_INVALID_ARG;
    pa_status st = check_pool_shape(num_kv_heads, head_dim, block_size, src_num_blocks, dtype, true);
    if (st != PA_OK) return st;
    if (!src_k || !src_v || !dst_k || !dst_v || !block_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v) ||
        !aligned8(block_mapping) || (d_status && !aligned4(d_status)))
        return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    const void *sk, *sv, *dk, *dv, *map;
    if (!device_address(src_k, &sk) || !device_address(src_v, &sv) ||
        !device_address(dst_k, &dk) || !device_address(dst_v, &dv) ||
        !device_address(block_mapping, &map))
        return PA_ERR_INVALID_ARG;
    const int elem_bytes = pool_elem_bytes(dtype);
    const int64_t block_vecs =
        static_cast<int64_t>(block_size) * num_kv_heads * head_dim * elem_bytes / 16;
    const int64_t per_cta = static_cast<int64_t>(kSwapThreads) * kSwapVecsPerThread;
    const int64_t chunks = (block_vecs + per_cta - 1) / per_cta;
    if (chunks > 65535) return PA_ERR_UNSUPPORTED;
    const int32_t same_pool = (src_k == dst_k && src_v == dst_v) ? 1 : 0;
    dim3 grid(num_pairs, 2, static_cast<unsigned>(chunks));
    return launch_overlapped(swap_blocks_kernel, grid, dim3(kSwapThreads), 0, stream,
                             static_cast<const uint4*>(sk), static_cast<const uint4*>(sv),
                             static_cast<uint4*>(const_cast<void*>(dk)),
                             static_cast<uint4*>(const_cast<void*>(dv)),
                             static_cast<const int64_t*>(map), num_pairs, block_vecs,
                             src_num_blocks, dst_num_blocks, same_pool, d_status);
}
