// decode_common.cuh -- what every paged decode kernel shares (sm_100a):
// the CTA shape (four warps), longest-first dispatch of the sequences, the
// prefetch of a warp's first block-table chunk, the fused cache write of a
// 16-bit row, the fixed-order merge of the four warps' (max, exp-sum,
// output), the "no result" store of a CTA whose copies timed out, and the
// split-context reduction kernel.  Included by paged_decode.cu.
//
// paged_decode_reduce_kernel: one CTA per (sequence, query head) with more
// than one partition merges the partitions with the blocked-softmax rule of
// "PagedAttention：大模型KV Cache分页管理优化实践" §5.1 applied to partitions:
//   M = max_p m_p,  w_p = l_p * 2^(m_p - M),  out = sum_p w_p Ohat_p / sum_p w_p.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "pa.h"
#include "pa_common.cuh"

namespace pa {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kReduceRowsPerCta = 4;

template <typename T, int D, int G>
__device__ __forceinline__ void write_zero_rows(T* out, int s, int kvh, int num_q_heads)
{
    T* row = out + (static_cast<int64_t>(s) * num_q_heads + kvh * G) * D;
    for (int i = threadIdx.x; i < G * D / 8; i += blockDim.x)
        reinterpret_cast<uint4*>(row)[i] = make_uint4(0, 0, 0, 0);
}

// Longest-first dispatch.  The CTAs of a grid start in blockIdx order, so
// when CTA z serves the z-th sequence in order of decreasing context length
// (ties by index), the long contexts start first and the last wave holds
// the short ones: the tail where few CTAs are left shrinks.  A batch in
// which adjacent sequences share their stored prefix (the same first
// physical block, as the beams of one prompt) keeps the grid order instead:
// there the CTAs of one group running together, reusing the shared blocks
// in L2, is worth more than the order.  Every thread of the CTA calls this
// before anything else uses `scratch` (num_seqs + 1 ints of shared memory,
// reused afterwards); needs num_seqs <= blockDim.x.  The mapping is a
// permutation, so each sequence is served exactly once; the work of a
// (sequence, head, partition) does not depend on which CTA runs it, so
// results are unchanged.
__device__ __forceinline__ int lpt_sequence(const int32_t* __restrict__ context_lens,
                                            const int32_t* __restrict__ block_tables,
                                            int32_t max_blocks_per_seq, int32_t num_seqs,
                                            int rank, int32_t* scratch)
{
    const int t = threadIdx.x;
    int32_t c = 0;
    bool shares = false;
    if (t < num_seqs) {
        c = context_lens[t];
        scratch[t] = c;
        if (t > 0)
            shares = block_tables[static_cast<int64_t>(t) * max_blocks_per_seq] ==
                     block_tables[static_cast<int64_t>(t - 1) * max_blocks_per_seq];
    }
    if (__syncthreads_or(shares)) return rank;   // grid order; scratch is not read again
    if (t < num_seqs) {
        int r = 0;
        for (int j = 0; j < num_seqs; ++j) {
            const int32_t cj = scratch[j];
            r += (cj > c || (cj == c && j < t)) ? 1 : 0;
        }
        if (r == rank) scratch[num_seqs] = t;
    }
    __syncthreads();
    const int pick = scratch[num_seqs];
    __syncthreads();   // scratch is free again
    return pick;
}

// A warp's first chunk of table entries (blocks warp + kWarps * lane of the
// partition), read before the context length is known: the index is checked
// against the table row only, so the load is in bounds whatever the context,
// and it overlaps the context-length load instead of following it.  Lanes
// past the warp's block count discard their entry.
__device__ __forceinline__ int prefetch_table_chunk(const int32_t* __restrict__ block_tables,
                                                    int s, int max_blocks_per_seq, int blk_begin,
                                                    int warp, int lane)
{
    const int idx = blk_begin + warp + kWarps * lane;
    return idx < max_blocks_per_seq
               ? block_tables[static_cast<int64_t>(s) * max_blocks_per_seq + idx]
               : -1;
}

// Fused append: the warp that loads the block holding a sequence's new token
// (position ctx - 1) first writes that token's K and V row for its kv head
// into the pools at the given physical block, then makes the writes visible
// to the tensor-copy engine before the block's tiles are requested.  No
// other warp or CTA reads that (token, kv head) row.  Warp-uniform; the
// caller issues the block's copies right after.
template <typename T, int D, int BS>
__device__ __forceinline__ void append_row_warp(
    const T* __restrict__ new_key, const T* __restrict__ new_value, T* __restrict__ k_cache,
    T* __restrict__ v_cache, int s, int kvh, int num_kv_heads, int32_t pos, int32_t phys,
    int lane)
{
    const int64_t slot = static_cast<int64_t>(phys) * BS + pos % BS;
    const int64_t src = (static_cast<int64_t>(s) * num_kv_heads + kvh) * D;
    const int64_t dst = (slot * num_kv_heads + kvh) * D;
    if (lane < D / 8) {
        const uint4 kv = ld_nc_v4(new_key + src + lane * 8);
        const uint4 vv = ld_nc_v4(new_value + src + lane * 8);
        *reinterpret_cast<uint4*>(k_cache + dst + lane * 8) = kv;
        *reinterpret_cast<uint4*>(v_cache + dst + lane * 8) = vv;
        fence_proxy_async_global();
    }
    __syncwarp();
    fence_proxy_async_global();
}

// The CTA's last step: merge the four warps' (max, exp-sum, output) for the
// G heads of its kv head in a fixed order, then either write the output row
// (context in one partition) or the partition's max, sum and normalised
// output to the workspace.  epi_o is [warp][g][D], epi_m / epi_l [warp][g],
// in shared memory, complete (the caller synchronised the CTA).
template <typename T, int D, int G>
__device__ __forceinline__ void merge_warps_and_store(
    const float* epi_o, const float* epi_m, const float* epi_l, T* __restrict__ out,
    float* __restrict__ ws_o, float2* __restrict__ ws_ml, int s, int kvh, int part, int nparts,
    int num_q_heads, int max_parts)
{
    for (int idx = threadIdx.x; idx < G * D / 8; idx += kThreads) {
        const int g = idx / (D / 8);
        const int d0 = (idx % (D / 8)) * 8;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, epi_m[w * G + g]);
        const float msub = M == -INFINITY ? 0.f : M;
        float L = 0.f;
        float O[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) O[e] = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float f = exp2f(epi_m[w * G + g] - msub);
            L = fmaf(f, epi_l[w * G + g], L);
            const float4* src = reinterpret_cast<const float4*>(epi_o + (w * G + g) * D + d0);
            const float4 a = src[0], b = src[1];
            O[0] = fmaf(f, a.x, O[0]); O[1] = fmaf(f, a.y, O[1]);
            O[2] = fmaf(f, a.z, O[2]); O[3] = fmaf(f, a.w, O[3]);
            O[4] = fmaf(f, b.x, O[4]); O[5] = fmaf(f, b.y, O[5]);
            O[6] = fmaf(f, b.z, O[6]); O[7] = fmaf(f, b.w, O[7]);
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) O[e] *= inv;
        const int h = kvh * G + g;
        const int64_t row = static_cast<int64_t>(s) * num_q_heads + h;
        if (nparts == 1) {
            *reinterpret_cast<uint4*>(out + row * D + d0) = pack8<T>(O);
        } else {
            const int64_t prow = row * max_parts + part;
            float4* dst = reinterpret_cast<float4*>(ws_o + prow * D + d0);
            dst[0] = make_float4(O[0], O[1], O[2], O[3]);
            dst[1] = make_float4(O[4], O[5], O[6], O[7]);
            if (d0 == 0) ws_ml[prow] = make_float2(M, L);
        }
    }
}

// The result of a CTA whose copies timed out is "nothing": zero output rows
// when the context is one partition, else an empty partial (max -inf, sum
// 0, zero output) that the reduction weighs with 0.  Global memory only:
// the CTA's shared memory may still be the target of copies in flight.
template <typename T, int D, int G>
__device__ __forceinline__ void store_aborted_rows(T* __restrict__ out, float* __restrict__ ws_o,
                                                   float2* __restrict__ ws_ml, int s, int kvh,
                                                   int part, int nparts, int num_q_heads,
                                                   int max_parts)
{
    for (int idx = threadIdx.x; idx < G * D / 8; idx += kThreads) {
        const int g = idx / (D / 8);
        const int d0 = (idx % (D / 8)) * 8;
        const int64_t row = static_cast<int64_t>(s) * num_q_heads + kvh * G + g;
        if (nparts == 1) {
            *reinterpret_cast<uint4*>(out + row * D + d0) = make_uint4(0, 0, 0, 0);
        } else {
            const int64_t prow = row * max_parts + part;
            float4* dst = reinterpret_cast<float4*>(ws_o + prow * D + d0);
            dst[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            dst[1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (d0 == 0) ws_ml[prow] = make_float2(-INFINITY, 0.f);
        }
    }
}


// The split-context reduction takes one of two shapes, chosen per launch
// from the number of partitions:
//   * many partitions (kWideRowParts or more): one CTA of kReduceWarps warps
//     per (sequence, query head); every warp weighs every kReduceWarps-th
//     partition, so a long context's partials are read by many warps at
//     once (one warp walking 64 partitions in sequence left the memory
//     system mostly idle: about 3.5 warps per SM on the long-context
//     workload);
//   * few partitions: one warp per (sequence, query head), four rows per
//     CTA, so short rows do not leave seven warps of a CTA idle.
// Either way every warp keeps the loads of four partitions in flight.
constexpr int kReduceWarps = 8;
constexpr int kWideRowParts = 16;

// Merge the partitions' (max, exp-sum, normalised output) of the rows whose
// context spans several partitions (rows of one partition were written by
// the decode kernel).  M = max_p m_p, w_p = l_p * 2^(m_p - M),
// out = sum_p w_p Ohat_p / sum_p w_p.  WPR = warps per row (1 or
// kReduceWarps); with several, the warps' sums are added in a fixed order,
// so the result is deterministic either way.
template <typename T, int D, int WPR>
__global__ void __launch_bounds__(WPR == 1 ? kReduceRowsPerCta * 32 : WPR * 32)
    paged_decode_reduce_kernel(T* __restrict__ out, const float* __restrict__ ws_o,
                               const float2* __restrict__ ws_ml,
                               const int32_t* __restrict__ context_lens, int32_t num_seqs,
                               int32_t num_q_heads, int32_t max_context_len,
                               int32_t max_blocks_per_seq, int32_t block_size,
                               int32_t partition_size, int32_t max_parts)
{
    grid_dependency_wait();
    constexpr int EPL = D / 32;     // elements per lane
    constexpr int kSmemWarps = WPR == 1 ? 1 : WPR;
    __shared__ float s_acc[kSmemWarps][D];
    __shared__ float s_w[kSmemWarps];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = WPR == 1 ? static_cast<int64_t>(blockIdx.x) * kReduceRowsPerCta + warp
                                 : static_cast<int64_t>(blockIdx.x);
    const int wr = WPR == 1 ? 0 : warp;             // this warp's place in its row
    if (row >= static_cast<int64_t>(num_seqs) * num_q_heads) return;
    const int s = static_cast<int>(row / num_q_heads);
    const int32_t ctx = context_lens[s];
    if (ctx <= 0 || ctx > max_context_len ||
        static_cast<int64_t>(ctx) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
        return;                                     // written by the first kernel
    const int np = (ctx + partition_size - 1) / partition_size;
    if (np <= 1) return;
    const float2* ml = ws_ml + row * max_parts;
    float M = -INFINITY;
    for (int p = lane; p < np; p += 32) M = fmaxf(M, ml[p].x);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, m));
    const float msub = M == -INFINITY ? 0.f : M;
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    float W = 0.f;
    const float* orow = ws_o + row * max_parts * D + lane * EPL;
    using Vec = typename std::conditional<EPL == 4, float4, float2>::type;
    auto weigh = [&](const float2 v, const Vec x) {
        const float w = v.y * exp2f(v.x - msub);
        W += w;
        const float* xf = reinterpret_cast<const float*>(&x);
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, xf[e], acc[e]);
    };
    // four of this warp's partitions per round, all their loads issued first
    constexpr int kBatch = 4;
    int p = wr;
    for (; p + (kBatch - 1) * WPR < np; p += kBatch * WPR) {
        float2 v[kBatch];
        Vec x[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int q = p + j * WPR;
            v[j] = ml[q];
            x[j] = *reinterpret_cast<const Vec*>(orow + static_cast<int64_t>(q) * D);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) weigh(v[j], x[j]);
    }
    for (; p < np; p += WPR)
        weigh(ml[p], *reinterpret_cast<const Vec*>(orow + static_cast<int64_t>(p) * D));
    if constexpr (WPR > 1) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) s_acc[warp][lane * EPL + e] = acc[e];
        if (lane == 0) s_w[warp] = W;
        __syncthreads();
        if (warp != 0) return;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        W = 0.f;
#pragma unroll
        for (int w = 0; w < WPR; ++w) {
            W += s_w[w];
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] += s_acc[w][lane * EPL + e];
        }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    T* dst = out + row * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; e += 2)
        *reinterpret_cast<uint32_t*>(dst + e) = Elem<T>::from_float2(acc[e] * inv, acc[e + 1] * inv);
}

}  // namespace pa
