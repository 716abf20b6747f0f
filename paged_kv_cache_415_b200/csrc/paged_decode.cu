// paged_decode.cu -- host entry points of single-query attention over a
// paged KV cache (sm_100a): argument checks, the partition choice, the
// tensor maps of the pools, the dispatch over (element type, head_dim,
// block_size, query group) to the kernel families, and their launches with
// programmatic dependent launch.
//
// The kernels live in headers of their own, one per family:
//   paged_decode_fp32.cuh    query groups G < 4, fp32 CUDA-core arithmetic;
//   paged_decode_mma.cuh     G >= 4, warp-level tensor-core contractions;
//   paged_decode_q8.cuh      pools of one-byte codes (e4m3 or int8);
//   paged_decode_shared.cuh  groups of sequences sharing a stored prefix;
//   decode_common.cuh        what they share, and the split-context
//                            reduction kernel.
//
// The whole computation has a fixed summation order, so results are
// deterministic and do not depend on where the blocks sit in the pool.
#include <cuda.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "pa.h"
#include "pa_common.cuh"
#include "pa_host.h"
#include "pa_selftest.h"
#include "decode_common.cuh"
#include "paged_decode_fp32.cuh"
#include "paged_decode_mma.cuh"
#include "paged_decode_shared.cuh"
#include "paged_decode_q8.cuh"
#include "paged_decode_q8_pair.cuh"

namespace pa {

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

struct DecodeArgs {
    void* out;
    const void* query;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    int32_t num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq;
    int64_t num_blocks;
    int32_t max_context_len;
    float scale_log2;
    int32_t partition_size, max_parts;
    float* ws_o;
    float2* ws_ml;
    int32_t* d_status;
    cudaStream_t stream;
    const void* new_key = nullptr;     // fused append (one token per sequence), or null
    const void* new_value = nullptr;
    int32_t lpt_seqs = 0;              // > 0: longest-first dispatch over this many sequences
    float k_inv = 1.f, v_inv = 1.f;    // quantised pools: reciprocal scales of the fused write
    uint32_t probe_us = 0;             // test hook of the bounded waits (pa_selftest_*); 0 = off
    float* k_scales = nullptr;         // row-scale pools of quantised K/V, or null (pool scales)
    float* v_scales = nullptr;
};

constexpr int kMaxDevices = 64;

// Streaming multiprocessors of the current device (queried once per device).
static int sm_count()
{
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < kMaxDevices) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < kMaxDevices) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

template <typename Kernel>
static bool ensure_smem_attr(Kernel kernel, int bytes, std::atomic<uint64_t>& done_mask)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
    if (bit && (done_mask.load(std::memory_order_relaxed) & bit)) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return false;
    done_mask.fetch_or(bit, std::memory_order_relaxed);
    return true;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link-time dependency on libcuda).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A pool [num_blocks][B][Hkv][D] of 16-bit elements as a 4-D tensor
// (innermost first: D, Hkv, B, num_blocks) whose box is one block of one kv
// head: D x 1 x B x 1, landing in shared memory as B dense rows of D.
static bool encode_pool_map(CUtensorMap* map, const void* pool, int32_t head_dim,
                            int32_t num_kv_heads, int32_t block_size, int64_t num_blocks)
{
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim),
                                static_cast<cuuint64_t>(num_kv_heads),
                                static_cast<cuuint64_t>(block_size),
                                static_cast<cuuint64_t>(num_blocks)};
    const cuuint64_t row = static_cast<cuuint64_t>(head_dim) * 2;
    const cuuint64_t strides[3] = {row, row * num_kv_heads, row * num_kv_heads * block_size};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(head_dim), 1u,
                               static_cast<cuuint32_t>(block_size), 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult res = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(pool), dims,
                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS;
}

// The same pool as a 5-D tensor (innermost first: 64 dims, B tokens, D/64
// halves, Hkv, num_blocks) whose box is one block of one kv head, stored in
// shared memory as [D/64][B][64] rows of 128 bytes with the 128-byte swizzle
// (16-byte chunk c of row r kept at chunk c ^ (r % 8)).
static bool encode_pool_map_swizzled(CUtensorMap* map, const void* pool, int32_t head_dim,
                                     int32_t num_kv_heads, int32_t block_size, int64_t num_blocks)
{
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(head_dim) * 2;
    const cuuint64_t dims[5] = {64u, static_cast<cuuint64_t>(block_size),
                                static_cast<cuuint64_t>(head_dim / 64),
                                static_cast<cuuint64_t>(num_kv_heads),
                                static_cast<cuuint64_t>(num_blocks)};
    const cuuint64_t strides[4] = {row * num_kv_heads, 128u, row, row * num_kv_heads * block_size};
    const cuuint32_t box[5] = {64u, static_cast<cuuint32_t>(block_size),
                               static_cast<cuuint32_t>(head_dim / 64), 1u, 1u};
    const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    const CUresult res = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 5, const_cast<void*>(pool), dims,
                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS;
}

// A pool [num_blocks][B][Hkv][D] of one-byte codes as a 4-D tensor whose
// box is one block of `heads` adjacent kv heads (1 or 2): B x heads rows of
// D bytes, with the 128-byte swizzle when a row is 128 bytes (else dense).
static bool encode_pool_map_q8(CUtensorMap* map, const void* pool, int32_t head_dim,
                                int32_t num_kv_heads, int32_t block_size, int64_t num_blocks,
                                uint32_t heads = 1u)
{
    const CUtensorMapSwizzle swz =
        head_dim == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim),
                                static_cast<cuuint64_t>(num_kv_heads),
                                static_cast<cuuint64_t>(block_size),
                                static_cast<cuuint64_t>(num_blocks)};
    const cuuint64_t row = static_cast<cuuint64_t>(head_dim);
    const cuuint64_t strides[3] = {row, row * num_kv_heads, row * num_kv_heads * block_size};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(head_dim), heads,
                               static_cast<cuuint32_t>(block_size), 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult res = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(pool), dims,
                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS;
}

// The split-context reduction after a decode launch whose contexts span
// several partitions: a CTA of kReduceWarps warps per (sequence, query head)
// when there are many partitions, else one warp per row.
template <typename T, int D>
static pa_status launch_reduce(const DecodeArgs& a)
{
    const int64_t rows = static_cast<int64_t>(a.num_seqs) * a.num_q_heads;
    if (a.max_parts >= kWideRowParts)
        return launch_overlapped(paged_decode_reduce_kernel<T, D, kReduceWarps>,
                                 dim3(static_cast<unsigned>(rows)), dim3(kReduceWarps * 32), 0,
                                 a.stream, static_cast<T*>(a.out), a.ws_o, a.ws_ml,
                                 a.context_lens, a.num_seqs, a.num_q_heads, a.max_context_len,
                                 a.max_blocks_per_seq, a.block_size, a.partition_size,
                                 a.max_parts);
    const unsigned ctas = static_cast<unsigned>((rows + kReduceRowsPerCta - 1) / kReduceRowsPerCta);
    return launch_overlapped(paged_decode_reduce_kernel<T, D, 1>, dim3(ctas),
                             dim3(kReduceRowsPerCta * 32), 0, a.stream, static_cast<T*>(a.out),
                             a.ws_o, a.ws_ml, a.context_lens, a.num_seqs, a.num_q_heads,
                             a.max_context_len, a.max_blocks_per_seq, a.block_size,
                             a.partition_size, a.max_parts);
}

// A CTA per pair of adjacent kv heads (one copy brings both heads' rows of a
// block, and each warp takes twice the blocks): with an even number of kv
// heads, when a CTA per kv head would give each warp fewer than
// kPairBelowBlocks blocks of its partition.  There the per-CTA prologue and
// epilogue weigh enough that twice the blocks per warp pays (long contexts
// in 512-token partitions: 8 blocks per warp); above it, the shorter CTAs of
// the per-head kernel balance ragged batches better.
constexpr int kPairBelowBlocks = 16;

template <typename Codes, typename T, int D, int BS, int G, bool ROWS>
static pa_status launch_decode_q8_pair(const DecodeArgs& a, float v_scale)
{
    using S = Q8PairShape<D, BS, G, ROWS>;
    static std::atomic<uint64_t> attr_done{0};
    auto kernel = std::is_same<Codes, Int8Codes>::value
                      ? paged_decode_int8_pair_kernel<T, D, BS, G, ROWS>
                      : paged_decode_fp8_pair_kernel<T, D, BS, G, ROWS>;
    if (!ensure_smem_attr(kernel, S::SMEM_BYTES, attr_done)) return PA_ERR_CUDA;
    CUtensorMap tm_k, tm_v;
    if (!encode_pool_map_q8(&tm_k, a.k_cache, D, a.num_kv_heads, BS, a.num_blocks, 2u) ||
        !encode_pool_map_q8(&tm_v, a.v_cache, D, a.num_kv_heads, BS, a.num_blocks, 2u))
        return PA_ERR_CUDA;
    dim3 grid(a.num_kv_heads / 2, a.max_parts, a.num_seqs);
    pa_status st = launch_overlapped(
        kernel, grid, dim3(kThreads), S::SMEM_BYTES, a.stream, tm_k, tm_v, static_cast<T*>(a.out),
        static_cast<const T*>(a.query), a.block_tables, a.context_lens, a.num_q_heads,
        a.max_blocks_per_seq, a.num_blocks, a.max_context_len, a.scale_log2, v_scale,
        a.partition_size, a.max_parts, a.ws_o, a.ws_ml, a.d_status, a.lpt_seqs,
        static_cast<const T*>(a.new_key), static_cast<const T*>(a.new_value),
        static_cast<uint8_t*>(const_cast<void*>(a.k_cache)),
        static_cast<uint8_t*>(const_cast<void*>(a.v_cache)), a.num_kv_heads, a.k_inv, a.v_inv,
        a.probe_us, a.k_scales, a.v_scales);
    if (st != PA_OK || a.max_parts <= 1) return st;
    return launch_reduce<T, D>(a);
}

template <typename Codes, typename T, int D, int BS, int G, bool ROWS>
static pa_status launch_decode_q8(const DecodeArgs& a, float v_scale)
{
    if (a.num_kv_heads % 2 == 0 && a.partition_size < kPairBelowBlocks * kWarps * BS)
        return launch_decode_q8_pair<Codes, T, D, BS, G, ROWS>(a, v_scale);
    using S = Q8Shape<D, BS, G, ROWS>;
    static std::atomic<uint64_t> attr_done{0};
    auto kernel = std::is_same<Codes, Int8Codes>::value
                      ? paged_decode_int8_kernel<T, D, BS, G, ROWS>
                      : paged_decode_fp8_kernel<T, D, BS, G, ROWS>;
    if (!ensure_smem_attr(kernel, S::SMEM_BYTES, attr_done)) return PA_ERR_CUDA;
    CUtensorMap tm_k, tm_v;
    if (!encode_pool_map_q8(&tm_k, a.k_cache, D, a.num_kv_heads, BS, a.num_blocks) ||
        !encode_pool_map_q8(&tm_v, a.v_cache, D, a.num_kv_heads, BS, a.num_blocks))
        return PA_ERR_CUDA;
    dim3 grid(a.num_kv_heads, a.max_parts, a.num_seqs);
    pa_status st = launch_overlapped(
        kernel, grid, dim3(kThreads), S::SMEM_BYTES, a.stream, tm_k, tm_v, static_cast<T*>(a.out),
        static_cast<const T*>(a.query), a.block_tables, a.context_lens, a.num_q_heads,
        a.max_blocks_per_seq, a.num_blocks, a.max_context_len, a.scale_log2, v_scale,
        a.partition_size, a.max_parts, a.ws_o, a.ws_ml, a.d_status, a.lpt_seqs,
        static_cast<const T*>(a.new_key), static_cast<const T*>(a.new_value),
        static_cast<uint8_t*>(const_cast<void*>(a.k_cache)),
        static_cast<uint8_t*>(const_cast<void*>(a.v_cache)), a.num_kv_heads, a.k_inv, a.v_inv,
        a.probe_us, a.k_scales, a.v_scales);
    if (st != PA_OK || a.max_parts <= 1) return st;
    return launch_reduce<T, D>(a);
}

template <typename Codes, typename T, int D, int BS, bool ROWS>
static pa_status dispatch_q8_group_rows(const DecodeArgs& a, float v_scale)
{
    switch (a.num_q_heads / a.num_kv_heads) {
    case 1: return launch_decode_q8<Codes, T, D, BS, 1, ROWS>(a, v_scale);
    case 2: return launch_decode_q8<Codes, T, D, BS, 2, ROWS>(a, v_scale);
    case 4: return launch_decode_q8<Codes, T, D, BS, 4, ROWS>(a, v_scale);
    case 8: return launch_decode_q8<Codes, T, D, BS, 8, ROWS>(a, v_scale);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename Codes, typename T, int D, int BS>
static pa_status dispatch_q8_group(const DecodeArgs& a, float v_scale)
{
    return a.k_scales != nullptr ? dispatch_q8_group_rows<Codes, T, D, BS, true>(a, v_scale)
                                 : dispatch_q8_group_rows<Codes, T, D, BS, false>(a, v_scale);
}

template <typename Codes, typename T>
static pa_status dispatch_q8(const DecodeArgs& a, float v_scale)
{
    const int32_t d = a.head_dim, b = a.block_size;
    if (d == 64 && b == 16) return dispatch_q8_group<Codes, T, 64, 16>(a, v_scale);
    if (d == 64 && b == 32) return dispatch_q8_group<Codes, T, 64, 32>(a, v_scale);
    if (d == 128 && b == 16) return dispatch_q8_group<Codes, T, 128, 16>(a, v_scale);
    if (d == 128 && b == 32) return dispatch_q8_group<Codes, T, 128, 32>(a, v_scale);
    return PA_ERR_UNSUPPORTED;
}

template <typename T, int D, int BS, int G>
static pa_status launch_decode(const DecodeArgs& a)
{
    // Grouped heads (G >= 4) in 16-token slices: tensor-core contractions.
    constexpr bool kMma = G >= 4 && BS % 16 == 0;
    dim3 grid(a.num_kv_heads, a.max_parts, a.num_seqs);
    CUtensorMap tm_k, tm_v;
    if constexpr (kMma) {
        using S = MmaShape<D, BS, G>;
        static std::atomic<uint64_t> attr_done{0};
        auto kernel = paged_decode_mma_kernel<T, D, BS, G>;
        if (!ensure_smem_attr(kernel, S::SMEM_BYTES, attr_done)) return PA_ERR_CUDA;
        if (!encode_pool_map_swizzled(&tm_k, a.k_cache, D, a.num_kv_heads, BS, a.num_blocks) ||
            !encode_pool_map_swizzled(&tm_v, a.v_cache, D, a.num_kv_heads, BS, a.num_blocks))
            return PA_ERR_CUDA;
        const pa_status ls = launch_overlapped(
            kernel, grid, dim3(kThreads), S::SMEM_BYTES, a.stream, tm_k, tm_v,
            static_cast<T*>(a.out), static_cast<const T*>(a.query), a.block_tables, a.context_lens,
            a.num_q_heads, a.max_blocks_per_seq, a.num_blocks, a.max_context_len, a.scale_log2,
            a.partition_size, a.max_parts, a.ws_o, a.ws_ml, a.d_status,
            static_cast<const T*>(a.new_key), static_cast<const T*>(a.new_value),
            static_cast<T*>(const_cast<void*>(a.k_cache)), static_cast<T*>(const_cast<void*>(a.v_cache)),
            a.num_kv_heads, a.lpt_seqs, a.probe_us);
        if (ls != PA_OK) return ls;
    } else {
        using S = DecodeShape<D, BS, G>;
        static std::atomic<uint64_t> attr_done{0};
        auto kernel = paged_decode_kernel<T, D, BS, G>;
        if (!ensure_smem_attr(kernel, S::SMEM_BYTES, attr_done)) return PA_ERR_CUDA;
        if (!encode_pool_map(&tm_k, a.k_cache, D, a.num_kv_heads, BS, a.num_blocks) ||
            !encode_pool_map(&tm_v, a.v_cache, D, a.num_kv_heads, BS, a.num_blocks))
            return PA_ERR_CUDA;
        const pa_status ls = launch_overlapped(
            kernel, grid, dim3(kThreads), S::SMEM_BYTES, a.stream, tm_k, tm_v,
            static_cast<T*>(a.out), static_cast<const T*>(a.query), a.block_tables, a.context_lens,
            a.num_q_heads, a.max_blocks_per_seq, a.num_blocks, a.max_context_len, a.scale_log2,
            a.partition_size, a.max_parts, a.ws_o, a.ws_ml, a.d_status,
            static_cast<const T*>(a.new_key), static_cast<const T*>(a.new_value),
            static_cast<T*>(const_cast<void*>(a.k_cache)), static_cast<T*>(const_cast<void*>(a.v_cache)),
            a.num_kv_heads, a.lpt_seqs, a.probe_us);
        if (ls != PA_OK) return ls;
    }
    if (a.max_parts <= 1) return PA_OK;
    return launch_reduce<T, D>(a);
}

template <typename T, int D, int BS>
static pa_status dispatch_group(const DecodeArgs& a)
{
    switch (a.num_q_heads / a.num_kv_heads) {
    case 1: return launch_decode<T, D, BS, 1>(a);
    case 2: return launch_decode<T, D, BS, 2>(a);
    case 4: return launch_decode<T, D, BS, 4>(a);
    case 8: return launch_decode<T, D, BS, 8>(a);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T, int D>
static pa_status dispatch_block(const DecodeArgs& a)
{
    switch (a.block_size) {
    case 8: return dispatch_group<T, D, 8>(a);
    case 16: return dispatch_group<T, D, 16>(a);
    case 32: return dispatch_group<T, D, 32>(a);
    default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T>
static pa_status dispatch_dim(const DecodeArgs& a)
{
    switch (a.head_dim) {
    case 64: return dispatch_block<T, 64>(a);
    case 128: return dispatch_block<T, 128>(a);
    default: return PA_ERR_UNSUPPORTED;
    }
}

struct SharedArgs {
    DecodeArgs d;
    const int32_t* prefix_lens;
    int32_t group_size, max_prefix_len, part_blocks;
};

template <typename T, int D, int BS>
static pa_status launch_shared(const SharedArgs& sa)
{
    using S = SharedShape<D, BS>;
    const DecodeArgs& a = sa.d;
    static std::atomic<uint64_t> attr_done{0};
    auto kernel = paged_decode_shared_kernel<T, D, BS>;
    if (!ensure_smem_attr(kernel, S::SMEM_BYTES, attr_done)) return PA_ERR_CUDA;
    CUtensorMap tm_k, tm_v;
    if (!encode_pool_map_swizzled(&tm_k, a.k_cache, D, a.num_kv_heads, BS, a.num_blocks) ||
        !encode_pool_map_swizzled(&tm_v, a.v_cache, D, a.num_kv_heads, BS, a.num_blocks))
        return PA_ERR_CUDA;
    const int32_t num_groups = a.num_seqs / sa.group_size;
    dim3 grid(a.num_kv_heads, a.max_parts, num_groups);
    pa_status st = launch_overlapped(
        kernel, grid, dim3(kThreads), S::SMEM_BYTES, a.stream, tm_k, tm_v, static_cast<T*>(a.out),
        static_cast<const T*>(a.query), a.block_tables, a.context_lens, sa.prefix_lens,
        sa.group_size, a.num_q_heads / a.num_kv_heads, a.num_q_heads, a.max_blocks_per_seq,
        a.num_blocks, a.max_context_len, sa.max_prefix_len, a.scale_log2, sa.part_blocks,
        a.max_parts, a.ws_o, a.ws_ml, a.d_status, a.probe_us);
    if (st != PA_OK || a.max_parts <= 1) return st;
    const int64_t rows = static_cast<int64_t>(a.num_seqs) * a.num_q_heads;
    const unsigned ctas = static_cast<unsigned>((rows + kReduceRowsPerCta - 1) / kReduceRowsPerCta);
    return launch_overlapped(paged_decode_shared_reduce_kernel<T, D>, dim3(ctas),
                             dim3(kReduceRowsPerCta * 32), 0, a.stream, static_cast<T*>(a.out),
                             a.ws_o, a.ws_ml, a.context_lens, sa.prefix_lens, a.num_seqs,
                             sa.group_size, a.num_q_heads, a.max_context_len, a.max_blocks_per_seq,
                             a.block_size, sa.max_prefix_len, sa.part_blocks, a.max_parts);
}

template <typename T>
static pa_status dispatch_shared(const SharedArgs& sa)
{
    const int32_t d = sa.d.head_dim, b = sa.d.block_size;
    if (d == 64 && b == 16) return launch_shared<T, 64, 16>(sa);
    if (d == 64 && b == 32) return launch_shared<T, 64, 32>(sa);
    if (d == 128 && b == 16) return launch_shared<T, 128, 16>(sa);
    if (d == 128 && b == 32) return launch_shared<T, 128, 32>(sa);
    return PA_ERR_UNSUPPORTED;
}

static bool supported_group(int32_t hq, int32_t hkv)
{
    if (hkv <= 0 || hq <= 0 || hq % hkv != 0) return false;
    const int32_t g = hq / hkv;
    return g == 1 || g == 2 || g == 4 || g == 8;
}

// Partition length: the caller's; else the whole (block-rounded) context
// when it is at most kMaxSinglePartition tokens and there are enough
// (sequence, kv head) pairs to fill the GPU on their own; else about a
// quarter of the longest context (so the longest sequences split into at
// least 4 CTAs), as a power of two between kMinPartition and
// kMaxPartition tokens (short enough to balance ragged contexts, long
// enough to amortise each CTA's start-up), halved while the grid would
// hold fewer than four CTAs per SM.  Fitted to partition sweeps of the
// Mistral-7B-shaped and long-context workloads on B200.
constexpr int kMinPartition = 512;
constexpr int kMaxPartition = 2048;
constexpr int kMaxSinglePartition = 2048;
constexpr int64_t kFillUnits = 888;    // 148 SMs x 3 CTAs x 2 waves
constexpr int64_t kFillSms = 148;

static int32_t choose_partition(int32_t num_seqs, int32_t num_kv_heads, int32_t block_size,
                                int32_t max_context_len, int32_t requested)
{
    if (requested > 0) return requested;
    const int32_t whole = max_context_len > 0
                              ? (max_context_len + block_size - 1) / block_size * block_size
                              : block_size;
    const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads;
    if (max_context_len <= kMaxSinglePartition && units >= kFillUnits) return whole;
    int32_t p = kMinPartition;
    while (p < kMaxPartition && p * 4 < max_context_len) p *= 2;
    // keep at least four CTAs per SM in the grid: halve while it is smaller
    const int64_t floor_ctas = 4 * static_cast<int64_t>(kFillSms);
    while (p > kMinPartition && units * ((max_context_len + p - 1) / p) < floor_ctas) p /= 2;
    p = p / block_size * block_size;
    return whole < p ? whole : p;
}

static size_t workspace_bytes_for(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                  int32_t max_parts)
{
    if (max_parts <= 1) return 0;
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * max_parts;
    return rows * head_dim * sizeof(float) + rows * sizeof(float2);
}

static int32_t parts_for(int32_t max_context_len, int32_t partition)
{
    return max_context_len <= 0 ? 1 : (max_context_len + partition - 1) / partition;
}

static pa_status check_decode_shape(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                    int32_t head_dim, int32_t block_size, int32_t max_context_len,
                                    int32_t partition_size)
{
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || max_context_len < 0 || partition_size < 0)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size) ||
        !supported_group(num_q_heads, num_kv_heads))
        return PA_ERR_UNSUPPORTED;
    if (partition_size % block_size != 0) return PA_ERR_INVALID_ARG;
    return PA_OK;
}

}  // namespace pa

extern "C" int32_t pa_paged_decode_partition_size(int32_t num_seqs, int32_t num_q_heads,
                                                  int32_t num_kv_heads, int32_t head_dim,
                                                  int32_t block_size, int32_t max_context_len,
                                                  int32_t partition_size)
{
    using namespace pa;
    if (check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                           max_context_len, partition_size) != PA_OK)
        return 0;
    return choose_partition(num_seqs, num_kv_heads, block_size, max_context_len, partition_size);
}

extern "C" size_t pa_paged_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                                 int32_t num_kv_heads, int32_t head_dim,
                                                 int32_t block_size, int32_t max_context_len,
                                                 int32_t partition_size)
{
    using namespace pa;
    if (check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                           max_context_len, partition_size) != PA_OK)
        return 0;
    const int32_t p = choose_partition(num_seqs, num_kv_heads, block_size, max_context_len,
                                       partition_size);
    return workspace_bytes_for(num_seqs, num_q_heads, head_dim, parts_for(max_context_len, p));
}

namespace pa {

// Element format of the K/V pools a decode call reads.
enum class KvCodes { kPlain, kE4m3, kInt8 };   // 16-bit elements, or one-byte codes

static pa_status decode_impl(void* out, const void* query, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                             int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq,
                             int64_t num_blocks, int32_t max_context_len, float scale,
                             int32_t partition_size, void* workspace, size_t workspace_bytes,
                             pa_dtype dtype, int32_t* d_status, pa_stream_t stream,
                             const void* new_key, const void* new_value,
                             KvCodes codes = KvCodes::kPlain, float k_scale = 1.f,
                             float v_scale = 1.f, uint32_t probe_us = 0,
                             float* k_scales = nullptr, float* v_scales = nullptr)
{
    pa_status st = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                      max_context_len, partition_size);
    if (st != PA_OK) return st;
    if (!supported_dtype(dtype)) return PA_ERR_UNSUPPORTED;
    if (max_blocks_per_seq <= 0 || num_blocks <= 0 || !isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (!out || !query || !k_cache || !v_cache || !block_tables || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(query) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned4(block_tables) || !aligned4(context_lens) || (d_status && !aligned4(d_status)))
        return PA_ERR_INVALID_ARG;
    if (new_key != nullptr &&
        (new_value == nullptr || !aligned16(new_key) || !aligned16(new_value)))
        return PA_ERR_INVALID_ARG;
    const bool quantised = codes != KvCodes::kPlain;
    const bool row_scaled = k_scales != nullptr || v_scales != nullptr;
    if (row_scaled && (!quantised || !k_scales || !v_scales || !aligned16(k_scales) ||
                 !aligned16(v_scales)))
        return PA_ERR_INVALID_ARG;
    if (quantised) {
        if (!(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(k_scale) || !isfinite(v_scale))
            return PA_ERR_INVALID_ARG;
        if (block_size % 16 != 0) return PA_ERR_UNSUPPORTED;
    }
    const int32_t partition = choose_partition(num_seqs, num_kv_heads, block_size, max_context_len,
                                               partition_size);
    const int32_t max_parts = parts_for(max_context_len, partition);
    const size_t need = workspace_bytes_for(num_seqs, num_q_heads, head_dim, max_parts);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
        return PA_ERR_INVALID_ARG;
    if (max_parts > 65535 || num_seqs > 65535) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;

    DecodeArgs a;
    a.out = out;
    a.query = query;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.head_dim = head_dim;
    a.block_size = block_size;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.max_context_len = max_context_len;
    a.scale_log2 = static_cast<float>(static_cast<double>(scale) * (quantised ? k_scale : 1.0) *
                                      1.4426950408889634);
    a.partition_size = partition;
    a.max_parts = max_parts;
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * max_parts;
    a.ws_o = need ? static_cast<float*>(workspace) : nullptr;
    a.ws_ml = need ? reinterpret_cast<float2*>(static_cast<char*>(workspace) +
                                               rows * head_dim * sizeof(float))
                   : nullptr;
    a.d_status = d_status;
    a.stream = stream;
    a.new_key = new_key;
    a.new_value = new_value;
    a.probe_us = probe_us;
    a.k_scales = k_scales;
    a.v_scales = v_scales;
    if (quantised) {
        a.k_inv = 1.0f / k_scale;      // the quantising write's fp32(1 / scale)
        a.v_inv = 1.0f / v_scale;
    }
    // Longest-first dispatch pays off once the grid spans more than about two
    // CTAs per SM (a tail exists) and the batch fits one CTA's threads.  Every
    // CTA ranks the batch itself (about num_seqs steps per thread), which is
    // small next to a whole context but not next to one partition of many:
    // with split contexts it is kept to small batches.
    const int64_t ctas = static_cast<int64_t>(num_kv_heads) * max_parts * num_seqs;
    if (num_seqs <= kThreads && ctas > 2 * static_cast<int64_t>(sm_count()) &&
        (max_parts == 1 || num_seqs <= 32))
        a.lpt_seqs = num_seqs;
    if (codes == KvCodes::kE4m3)
        return dtype == PA_DTYPE_F16 ? dispatch_q8<E4m3Codes, __half>(a, v_scale)
                                     : dispatch_q8<E4m3Codes, __nv_bfloat16>(a, v_scale);
    if (codes == KvCodes::kInt8)
        return dtype == PA_DTYPE_F16 ? dispatch_q8<Int8Codes, __half>(a, v_scale)
                                     : dispatch_q8<Int8Codes, __nv_bfloat16>(a, v_scale);
    return dtype == PA_DTYPE_F16 ? dispatch_dim<__half>(a) : dispatch_dim<__nv_bfloat16>(a);
}

}  // namespace pa

extern "C" pa_status pa_paged_decode(void* out, const void* query, const void* k_cache,
                                     const void* v_cache, const int32_t* block_tables,
                                     const int32_t* context_lens, int32_t num_seqs,
                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int32_t max_blocks_per_seq,
                                     int64_t num_blocks, int32_t max_context_len, float scale,
                                     int32_t partition_size, void* workspace,
                                     size_t workspace_bytes, pa_dtype dtype, int32_t* d_status,
                                     pa_stream_t stream)
{
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, nullptr, nullptr);
}

extern "C" pa_status pa_paged_decode_fp8(void* out, const void* query, const void* k_cache,
                                         const void* v_cache, const int32_t* block_tables,
                                         const int32_t* context_lens, int32_t num_seqs,
                                         int32_t num_q_heads, int32_t num_kv_heads,
                                         int32_t head_dim, int32_t block_size,
                                         int32_t max_blocks_per_seq, int64_t num_blocks,
                                         int32_t max_context_len, float scale, float k_scale,
                                         float v_scale, int32_t partition_size, void* workspace,
                                         size_t workspace_bytes, pa_dtype dtype,
                                         int32_t* d_status, pa_stream_t stream)
{
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, nullptr, nullptr,
                           pa::KvCodes::kE4m3, k_scale, v_scale);
}

extern "C" pa_status pa_paged_decode_fp8_append(
    void* out, const void* query, const void* key, const void* value, void* k_cache,
    void* v_cache, const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len, float scale,
    float k_scale, float v_scale, int32_t partition_size, void* workspace, size_t workspace_bytes,
    pa_dtype dtype, int32_t* d_status, pa_stream_t stream)
{
    if (key == nullptr || value == nullptr) return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, key, value,
                           pa::KvCodes::kE4m3, k_scale, v_scale);
}

extern "C" pa_status pa_paged_decode_int8(void* out, const void* query, const void* k_cache,
                                          const void* v_cache, const int32_t* block_tables,
                                          const int32_t* context_lens, int32_t num_seqs,
                                          int32_t num_q_heads, int32_t num_kv_heads,
                                          int32_t head_dim, int32_t block_size,
                                          int32_t max_blocks_per_seq, int64_t num_blocks,
                                          int32_t max_context_len, float scale, float k_scale,
                                          float v_scale, int32_t partition_size, void* workspace,
                                          size_t workspace_bytes, pa_dtype dtype,
                                          int32_t* d_status, pa_stream_t stream)
{
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, nullptr, nullptr,
                           pa::KvCodes::kInt8, k_scale, v_scale);
}

extern "C" pa_status pa_paged_decode_int8_append(
    void* out, const void* query, const void* key, const void* value, void* k_cache,
    void* v_cache, const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len, float scale,
    float k_scale, float v_scale, int32_t partition_size, void* workspace, size_t workspace_bytes,
    pa_dtype dtype, int32_t* d_status, pa_stream_t stream)
{
    if (key == nullptr || value == nullptr) return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, key, value,
                           pa::KvCodes::kInt8, k_scale, v_scale);
}

extern "C" pa_status pa_paged_decode_fp8_rowscale(
    void* out, const void* query, const void* k_cache, const void* v_cache, const float* k_scales,
    const float* v_scales, const int32_t* block_tables, const int32_t* context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float scale, int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
    int32_t* d_status, pa_stream_t stream)
{
    if (k_scales == nullptr || v_scales == nullptr) return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, nullptr, nullptr,
                           pa::KvCodes::kE4m3, 1.f, 1.f, 0u, const_cast<float*>(k_scales),
                           const_cast<float*>(v_scales));
}

extern "C" pa_status pa_paged_decode_fp8_rowscale_append(
    void* out, const void* query, const void* key, const void* value, void* k_cache,
    void* v_cache, float* k_scales, float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, float scale, int32_t partition_size, void* workspace,
    size_t workspace_bytes, pa_dtype dtype, int32_t* d_status, pa_stream_t stream)
{
    if (key == nullptr || value == nullptr || k_scales == nullptr || v_scales == nullptr)
        return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, key, value,
                           pa::KvCodes::kE4m3, 1.f, 1.f, 0u, k_scales, v_scales);
}

extern "C" pa_status pa_paged_decode_int8_rowscale(
    void* out, const void* query, const void* k_cache, const void* v_cache, const float* k_scales,
    const float* v_scales, const int32_t* block_tables, const int32_t* context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    float scale, int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
    int32_t* d_status, pa_stream_t stream)
{
    if (k_scales == nullptr || v_scales == nullptr) return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, nullptr, nullptr,
                           pa::KvCodes::kInt8, 1.f, 1.f, 0u, const_cast<float*>(k_scales),
                           const_cast<float*>(v_scales));
}

extern "C" pa_status pa_paged_decode_int8_rowscale_append(
    void* out, const void* query, const void* key, const void* value, void* k_cache,
    void* v_cache, float* k_scales, float* v_scales, const int32_t* block_tables,
    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, float scale, int32_t partition_size, void* workspace,
    size_t workspace_bytes, pa_dtype dtype, int32_t* d_status, pa_stream_t stream)
{
    if (key == nullptr || value == nullptr || k_scales == nullptr || v_scales == nullptr)
        return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, key, value,
                           pa::KvCodes::kInt8, 1.f, 1.f, 0u, k_scales, v_scales);
}

extern "C" pa_status pa_paged_decode_append(void* out, const void* query, const void* key,
                                            const void* value, void* k_cache, void* v_cache,
                                            const int32_t* block_tables,
                                            const int32_t* context_lens, int32_t num_seqs,
                                            int32_t num_q_heads, int32_t num_kv_heads,
                                            int32_t head_dim, int32_t block_size,
                                            int32_t max_blocks_per_seq, int64_t num_blocks,
                                            int32_t max_context_len, float scale,
                                            int32_t partition_size, void* workspace,
                                            size_t workspace_bytes, pa_dtype dtype,
                                            int32_t* d_status, pa_stream_t stream)
{
    if (key == nullptr || value == nullptr) return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, workspace,
                           workspace_bytes, dtype, d_status, stream, key, value);
}

// ---------------------------------------------------------------------------
// Shared-prefix decode
// ---------------------------------------------------------------------------
namespace pa {

static pa_status check_shared_shape(int32_t num_seqs, int32_t group_size, int32_t num_q_heads,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                    int32_t max_context_len, int32_t max_prefix_len,
                                    int32_t partition_size)
{
    pa_status st = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                      max_context_len, partition_size);
    if (st != PA_OK) return st;
    if (group_size <= 0 || num_seqs % group_size != 0 || max_prefix_len < 0 ||
        max_prefix_len > max_context_len)
        return PA_ERR_INVALID_ARG;
    if (block_size % 16 != 0 || group_size * (num_q_heads / num_kv_heads) > kSharedRows)
        return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

// The shared-prefix path splits each group's block list (prefix blocks, then
// every member's own): its partition is chosen as for a context as long as
// the longest list can be (group_size x the longest context), over the
// groups.  Returns the parts of the longest list.
static int32_t shared_parts(int32_t num_seqs, int32_t group_size, int32_t num_kv_heads,
                            int32_t block_size, int32_t max_context_len, int32_t partition_size,
                            int32_t* part_blocks)
{
    const int64_t list_tokens = static_cast<int64_t>(group_size) * max_context_len;
    const int32_t span = list_tokens > (1 << 30) ? (1 << 30) : static_cast<int32_t>(list_tokens);
    const int32_t partition = choose_partition(num_seqs / group_size, num_kv_heads, block_size,
                                               span, partition_size);
    *part_blocks = partition / block_size;
    const int64_t max_blocks = static_cast<int64_t>(group_size) *
                               ((max_context_len + block_size - 1) / block_size);
    const int64_t parts = (max_blocks + *part_blocks - 1) / *part_blocks;
    return static_cast<int32_t>(parts < 1 ? 1 : parts > (1 << 30) ? (1 << 30) : parts);
}

}  // namespace pa

extern "C" size_t pa_paged_decode_shared_prefix_workspace_size(
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_context_len, int32_t max_prefix_len,
    int32_t partition_size)
{
    using namespace pa;
    if (check_shared_shape(num_seqs, group_size, num_q_heads, num_kv_heads, head_dim, block_size,
                           max_context_len, max_prefix_len, partition_size) != PA_OK)
        return 0;
    int32_t part_blocks;
    const int32_t parts = shared_parts(num_seqs, group_size, num_kv_heads, block_size,
                                       max_context_len, partition_size, &part_blocks);
    if (parts <= 1) return 0;
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * parts;
    return rows * head_dim * sizeof(float) + rows * sizeof(float2);
}

namespace pa {

static pa_status shared_prefix_impl(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* prefix_lens,
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, int32_t max_prefix_len, float scale, int32_t partition_size,
    void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* d_status, pa_stream_t stream,
    uint32_t probe_us)
{
    pa_status st = check_shared_shape(num_seqs, group_size, num_q_heads, num_kv_heads, head_dim,
                                      block_size, max_context_len, max_prefix_len, partition_size);
    if (st != PA_OK) return st;
    if (!supported_dtype(dtype)) return PA_ERR_UNSUPPORTED;
    if (max_blocks_per_seq <= 0 || num_blocks <= 0 || !isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (!out || !query || !k_cache || !v_cache || !block_tables || !context_lens || !prefix_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(query) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned4(block_tables) || !aligned4(context_lens) || !aligned4(prefix_lens) ||
        (d_status && !aligned4(d_status)))
        return PA_ERR_INVALID_ARG;
    int32_t part_blocks;
    const int32_t parts = shared_parts(num_seqs, group_size, num_kv_heads, block_size,
                                       max_context_len, partition_size, &part_blocks);
    const size_t need = pa_paged_decode_shared_prefix_workspace_size(
        num_seqs, group_size, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
        max_prefix_len, partition_size);
    if (num_seqs == 0) return PA_OK;
    if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
        return PA_ERR_INVALID_ARG;
    if (num_seqs / group_size > 65535 || parts > 65535) return PA_ERR_UNSUPPORTED;

    SharedArgs sa;
    DecodeArgs& a = sa.d;
    a.out = out;
    a.query = query;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.head_dim = head_dim;
    a.block_size = block_size;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.max_context_len = max_context_len;
    a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    a.partition_size = part_blocks * block_size;
    a.max_parts = parts;
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * parts;
    a.ws_o = need > 0 ? static_cast<float*>(workspace) : nullptr;
    a.ws_ml = need > 0 ? reinterpret_cast<float2*>(static_cast<char*>(workspace) +
                                                   rows * head_dim * sizeof(float))
                       : nullptr;
    a.d_status = d_status;
    a.stream = stream;
    sa.prefix_lens = prefix_lens;
    sa.group_size = group_size;
    sa.max_prefix_len = max_prefix_len;
    sa.part_blocks = part_blocks;
    a.probe_us = probe_us;
    return dtype == PA_DTYPE_F16 ? dispatch_shared<__half>(sa) : dispatch_shared<__nv_bfloat16>(sa);
}

}  // namespace pa

extern "C" pa_status pa_paged_decode_shared_prefix(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* prefix_lens,
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, int32_t max_prefix_len, float scale, int32_t partition_size,
    void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* d_status, pa_stream_t stream)
{
    return pa::shared_prefix_impl(out, query, k_cache, v_cache, block_tables, context_lens,
                                  prefix_lens, num_seqs, group_size, num_q_heads, num_kv_heads,
                                  head_dim, block_size, max_blocks_per_seq, num_blocks,
                                  max_context_len, max_prefix_len, scale, partition_size, workspace,
                                  workspace_bytes, dtype, d_status, stream, 0u);
}

// ---------------------------------------------------------------------------
// Test entry points of the bounded waits (declared in pa_selftest.h): the
// decode kernels with every warp's first wait sent to an mbarrier that
// nothing completes, so the timeout and the abort path run for real.
// ---------------------------------------------------------------------------
static constexpr uint32_t kMaxProbeUs = 1000000u;   // longest probe wait: 1 s

extern "C" pa_status pa_selftest_decode_abort(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len, float scale,
    int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
    pa_dtype kv_dtype, uint32_t wait_limit_us, int32_t* d_status, pa_stream_t stream)
{
    using namespace pa;
    if (wait_limit_us == 0u || wait_limit_us > kMaxProbeUs) return PA_ERR_INVALID_ARG;
    KvCodes codes;
    if (kv_dtype == dtype) codes = KvCodes::kPlain;
    else if (kv_dtype == PA_DTYPE_FP8_E4M3) codes = KvCodes::kE4m3;
    else if (kv_dtype == PA_DTYPE_INT8) codes = KvCodes::kInt8;
    else return PA_ERR_UNSUPPORTED;
    return decode_impl(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                       num_blocks, max_context_len, scale, partition_size, workspace,
                       workspace_bytes, dtype, d_status, stream, nullptr, nullptr, codes, 1.f, 1.f,
                       wait_limit_us);
}

extern "C" pa_status pa_selftest_shared_prefix_abort(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* prefix_lens,
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, int32_t max_prefix_len, float scale, int32_t partition_size,
    void* workspace, size_t workspace_bytes, pa_dtype dtype, uint32_t wait_limit_us,
    int32_t* d_status, pa_stream_t stream)
{
    if (wait_limit_us == 0u || wait_limit_us > kMaxProbeUs) return PA_ERR_INVALID_ARG;
    return pa::shared_prefix_impl(out, query, k_cache, v_cache, block_tables, context_lens,
                                  prefix_lens, num_seqs, group_size, num_q_heads, num_kv_heads,
                                  head_dim, block_size, max_blocks_per_seq, num_blocks,
                                  max_context_len, max_prefix_len, scale, partition_size, workspace,
                                  workspace_bytes, dtype, d_status, stream, wait_limit_us);
}

// ---------------------------------------------------------------------------
// pa_paged_decode_no_alloc: the same decode with its split-context scratch in
// a file-scope device array instead of caller memory.
// ---------------------------------------------------------------------------
namespace pa {

static __device__ __align__(256) unsigned char g_no_alloc_workspace[PA_NO_ALLOC_WORKSPACE_BYTES];

// Device address of the array in the current context.  Looked up on every
// call (host code may not use the symbol itself as a device pointer), so
// that a cudaDeviceReset or another context on the device never leaves a
// stale address behind; after the first call on a device the lookup only
// reads the loaded module's table.
static pa_status no_alloc_workspace(void** ptr)
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_no_alloc_workspace) != cudaSuccess || p == nullptr)
        return PA_ERR_CUDA;
    *ptr = p;
    return PA_OK;
}

}  // namespace pa

extern "C" pa_status pa_paged_decode_no_alloc(void* out, const void* query, const void* k_cache,
                                              const void* v_cache, const int32_t* block_tables,
                                              const int32_t* context_lens, int32_t num_seqs,
                                              int32_t num_q_heads, int32_t num_kv_heads,
                                              int32_t head_dim, int32_t block_size,
                                              int32_t max_blocks_per_seq, int64_t num_blocks,
                                              int32_t max_context_len, float scale,
                                              int32_t partition_size, pa_dtype dtype,
                                              int32_t* d_status, pa_stream_t stream)
{
    using namespace pa;
    pa_status st = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                      max_context_len, partition_size);
    if (st != PA_OK) return st;
    const size_t need = pa_paged_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                                                       head_dim, block_size, max_context_len,
                                                       partition_size);
    if (need > PA_NO_ALLOC_WORKSPACE_BYTES) return PA_ERR_INVALID_ARG;
    // pointer checks before the array's address is looked up
    if (!out || !query || !k_cache || !v_cache || !block_tables || !context_lens ||
        !aligned16(out) || !aligned16(query) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned4(block_tables) || !aligned4(context_lens) || (d_status && !aligned4(d_status)))
        return PA_ERR_INVALID_ARG;
    void* ws = nullptr;
    if (need > 0) {
        st = no_alloc_workspace(&ws);
        if (st != PA_OK) return st;
    }
    return pa_paged_decode(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, max_context_len, scale, partition_size, ws,
                           need > 0 ? PA_NO_ALLOC_WORKSPACE_BYTES : 0, dtype, d_status, stream);
}
