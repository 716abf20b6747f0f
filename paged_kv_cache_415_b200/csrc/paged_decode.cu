// paged_decode.cu -- single-query attention over a paged KV cache (sm_100a).
//
// Kernel 1, paged_decode_kernel (query groups G < 4): one CTA per (kv head,
// context partition, sequence).  The CTA carries the G = Hq / Hkv query heads
// of its kv head, so every K/V byte is read from HBM once for all of them.
// Each of its four warps runs its own pipeline over every fourth physical
// block of the partition:
//   * the warp's block-table entries sit one per lane (32 blocks per load,
//     the first chunk read together with the context length) and are
//     broadcast with a shuffle ("PagedAttention：大模型KV Cache分页管理优化实践"
//     §3.2: flattened table, warp-level prefetch);
//   * one lane requests each block's K and V tile of this kv head (block_size
//     rows of head_dim elements) with two TMA tensor copies into the warp's
//     shared-memory ring of NSTAGE stages, completion counted on one mbarrier
//     per stage, so the next blocks are in flight while one is computed
//     (§4.2 prefetch, §5.2 overlap of copy and compute);
//   * scores q.k in fp32 (fma.rn.f32 on the 16-bit operands): 8 (or 16)
//     lanes share a token row and the partial dot products are reduced with
//     a transposing butterfly of warp shuffles; scale * log2(e) multiplies
//     the reduced score, so the exponentials are exp2;
//   * the softmax is the blocked form of §5.1 (分块Softmax算法) run online:
//     per tile the local max, the running (global) max, the exp-sum rescaled
//     to it, then the weighted V rows accumulate into fp32 outputs rescaled
//     the same way.
// At the end the four warps' (max, sum, output) are merged through shared
// memory in a fixed order.  A sequence whose context fits one partition gets
// its output row written directly; otherwise the partition's max, sum and
// normalised output go to the workspace.  With a fused append, the warp that
// loads the block holding a sequence's new token writes that token's K/V row
// first.  Small batches are dispatched longest context first (lpt_sequence).
//
// Kernel 2, paged_decode_reduce_kernel: one warp per (sequence, query head)
// with more than one partition merges the partitions with the same rule:
//   M = max_p m_p,  w_p = l_p * 2^(m_p - M),  out = sum_p w_p Ohat_p / sum_p w_p.
//
// The grouped-head (paged_decode_mma.cuh), one-byte-code (e4m3 or int8:
// paged_decode_q8.cuh) and shared-prefix (paged_decode_shared.cuh) kernels are included below; this
// file also holds the host entry points and their launch logic.
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

namespace pa {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kReduceRowsPerCta = 4;

template <int D, int BS, int G>
struct DecodeShape {
    static constexpr int LPT = (G >= 4 && D == 128) ? 16 : 8;   // lanes per token row
    static constexpr int RPW = 32 / LPT;                        // token rows per warp pass
    static constexpr int EPT = D / LPT;                         // elements per lane
    static constexpr int NCHUNK = EPT / 8;                      // 16-byte chunks per lane
    // Tokens scored per softmax step: the whole block, or a slice of it so
    // that a lane never holds more than 16 partial scores.
    static constexpr int CT_MAX = 16 * RPW / G > RPW ? 16 * RPW / G : RPW;
    static constexpr int CT = BS < CT_MAX ? BS : CT_MAX;
    static constexpr int TILES = BS / CT;
    static constexpr int ITERS = CT / RPW;                      // passes per tile
    static constexpr int ROW_BYTES = D * 2;
    static constexpr int TILE_BYTES = BS * ROW_BYTES;           // K (or V) of one block, one head
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int NSTAGE = STAGE_BYTES <= 4096 ? 3 : 2;
    static constexpr int NVAL = ITERS * G;                      // partial scores per lane
    static constexpr int NHELD = NVAL >= LPT ? NVAL / LPT : 1;  // scores per lane after reduce
    static constexpr int SM_TPL = (CT * G + 31) / 32;           // softmax items per lane
    static constexpr int WARP_STAGE_BYTES = NSTAGE * STAGE_BYTES;
    static constexpr int OFF_SCORES = kWarps * WARP_STAGE_BYTES;
    static constexpr int SCORE_FLOATS = CT * G;
    static constexpr int OFF_CORR = OFF_SCORES + kWarps * SCORE_FLOATS * 4;
    static constexpr int CORR_FLOATS = (G + 3) / 4 * 4;
    static constexpr int OFF_BARS = OFF_CORR + kWarps * CORR_FLOATS * 4;
    static constexpr int SMEM_BYTES = OFF_BARS + kWarps * NSTAGE * 8;
    static constexpr int EPI_BYTES = kWarps * G * (D + 2) * 4;
    // CTAs per SM the register budget is sized for: larger groups keep more
    // live state per lane (q and the output accumulators of every head).
    static constexpr int MIN_CTAS = G >= 8 ? 2 : 3;
    static_assert(EPI_BYTES <= OFF_SCORES, "epilogue must fit in the stage buffers");
    static_assert(EPT % 8 == 0, "lanes hold whole 16-byte chunks");
    static_assert(CT % RPW == 0 && BS % CT == 0, "tiles split evenly over the warp");
    static_assert(32 % G == 0, "group size divides the warp");
    static_assert(NVAL <= 16, "partial scores per lane");
};

// Sums NVAL per-lane partial values over groups of LPT lanes.  Each halving
// step sends the half of the values this lane does not keep and adds the
// partner's copy of the half it keeps, so the shuffle count falls from
// NVAL*log2(LPT) to about NVAL.  Returns the index of the first value the
// lane now holds in full; it holds NHELD consecutive values.
template <int NVAL, int LPT>
__device__ __forceinline__ int transpose_reduce(float (&v)[NVAL], int c)
{
    int base = 0;
    int n = NVAL;
#pragma unroll
    for (int m = LPT / 2; m >= 1; m >>= 1) {
        if (n > 1) {
            const bool upper = (c & m) != 0;
            const int half = n / 2;
#pragma unroll
            for (int j = 0; j < NVAL / 2; ++j) {
                if (j < half) {
                    const float lo = v[j], hi = v[j + half];
                    const float send = upper ? lo : hi;
                    const float keep = upper ? hi : lo;
                    v[j] = keep + __shfl_xor_sync(kFullMask, send, m);
                }
            }
            if (upper) base += half;
            n = half;
        } else {
            v[0] += __shfl_xor_sync(kFullMask, v[0], m);
        }
    }
    return base;
}

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

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(kThreads, (DecodeShape<D, BS, G>::MIN_CTAS)) paged_decode_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    T* __restrict__ out, const T* __restrict__ query, const int32_t* __restrict__ block_tables,
    const int32_t* __restrict__ context_lens, int32_t num_q_heads, int32_t max_blocks_per_seq,
    int64_t num_blocks, int32_t max_context_len, float scale_log2, int32_t partition_size,
    int32_t max_parts, float* __restrict__ ws_o, float2* __restrict__ ws_ml, int32_t* d_status,
    const T* __restrict__ new_key, const T* __restrict__ new_value, T* __restrict__ k_cache,
    T* __restrict__ v_cache, int32_t num_kv_heads, int32_t lpt_seqs)
{
    grid_dependency_wait();   // before any global access (see pa_common.cuh)
    using S = DecodeShape<D, BS, G>;
    constexpr int EP = S::EPT / 2;      // element pairs per lane
    extern __shared__ __align__(128) unsigned char smem[];

    const int kvh = blockIdx.x;
    const int part = blockIdx.y;
    const int s = lpt_seqs > 0
                      ? lpt_sequence(context_lens, block_tables, max_blocks_per_seq, lpt_seqs,
                                     blockIdx.z, reinterpret_cast<int32_t*>(smem))
                      : static_cast<int>(blockIdx.z);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int c = lane % S::LPT;        // position within the token row
    const int r = lane / S::LPT;        // token row within a pass

    const int pre_tbl = prefetch_table_chunk(block_tables, s, max_blocks_per_seq,
                                             blockIdx.y * partition_size / BS, warp, lane);
    const int32_t ctx = context_lens[s];
    if (ctx < 0 || ctx > max_context_len ||
        static_cast<int64_t>(ctx) > static_cast<int64_t>(max_blocks_per_seq) * BS) {
        if (part == 0) {
            write_zero_rows<T, D, G>(out, s, kvh, num_q_heads);
            if (threadIdx.x == 0) status_or(d_status, PA_STATUS_BAD_CONTEXT);
        }
        return;
    }
    if (ctx == 0) {
        if (part == 0) write_zero_rows<T, D, G>(out, s, kvh, num_q_heads);
        return;
    }
    const int tok_begin = part * partition_size;
    if (tok_begin >= ctx) return;
    const int tok_end = min(ctx, tok_begin + partition_size);
    const int nparts = (ctx + partition_size - 1) / partition_size;
    const int blk_begin = tok_begin / BS;
    const int nblk = (tok_end - tok_begin + BS - 1) / BS;
    const int nk = warp < nblk ? (nblk - warp + kWarps - 1) / kWarps : 0;   // this warp's blocks
    // the block (of this partition) holding the new token, when appending
    const int append_blk = (new_key != nullptr && part == nparts - 1) ? (ctx - 1) / BS - blk_begin : -1;

    unsigned char* wstage = smem + warp * S::WARP_STAGE_BYTES;
    float* wscore = reinterpret_cast<float*>(smem + S::OFF_SCORES) + warp * S::SCORE_FLOATS;
    float* wcorr = reinterpret_cast<float*>(smem + S::OFF_CORR) + warp * S::CORR_FLOATS;
    uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + S::OFF_BARS) + warp * S::NSTAGE;

    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < S::NSTAGE; ++st) mbar_init(&wbar[st], 1);
        fence_barrier_init();
    }
    __syncwarp();

    const int32_t* table = block_tables + static_cast<int64_t>(s) * max_blocks_per_seq + blk_begin;
    // The warp's k-th block is block warp + kWarps * k of the partition; one
    // table entry per lane, 32 blocks per load.
    auto load_table = [&](int chunk) -> int {
        const int kk = chunk * 32 + lane;
        return kk < nk ? table[warp + kWarps * kk] : -1;
    };
    int prod_chunk = 0, cons_chunk = 0;
    int prod_tbl = lane < nk ? pre_tbl : -1;   // load_table(0), already in flight
    int cons_tbl = prod_tbl;

    auto block_tokens = [&](int k) -> int {   // valid tokens of the warp's k-th block
        const int t0 = tok_begin + (warp + kWarps * k) * BS;
        return min(BS, tok_end - t0);
    };

    // Producer: one lane starts the two tensor copies (the K and V tiles of
    // this kv head: BS rows of D elements) of block k into its stage.
    auto issue = [&](int k) {
        const int chunk = k >> 5;
        if (chunk != prod_chunk) {
            prod_tbl = load_table(chunk);
            prod_chunk = chunk;
        }
        const int phys = __shfl_sync(kFullMask, prod_tbl, k & 31);
        if (warp + kWarps * k == append_blk) {
            if (phys >= 0 && static_cast<int64_t>(phys) < num_blocks)
                append_row_warp<T, D, BS>(new_key, new_value, k_cache, v_cache, s, kvh,
                                          num_kv_heads, ctx - 1, phys, lane);
            else if (lane == 0)
                status_or(d_status, PA_STATUS_BAD_SLOT);
        }
        if (lane == 0) {
            const int st = k % S::NSTAGE;
            const bool ok = phys >= 0 && static_cast<int64_t>(phys) < num_blocks;
            fence_proxy_async_smem();
            if (ok) {
                mbar_arrive_expect_tx(&wbar[st], 2u * S::TILE_BYTES);
                unsigned char* dst = wstage + st * S::STAGE_BYTES;
                tma_load_4d(dst, &tm_k, 0, kvh, 0, phys, &wbar[st]);
                tma_load_4d(dst + S::TILE_BYTES, &tm_v, 0, kvh, 0, phys, &wbar[st]);
            } else {
                status_or(d_status, PA_STATUS_BAD_BLOCK);
                mbar_arrive_expect_tx(&wbar[st], 0u);
            }
        }
    };

    const int prologue = min(nk, S::NSTAGE);
    for (int k = 0; k < prologue; ++k) issue(k);
    int issued = prologue;

    // q of every head in the group, this lane's elements, kept as the raw
    // 16-bit input pairs (the products with K are exact in fp32; the scale
    // is applied to the reduced scores).
    uint32_t qw[G][EP];
    {
        const T* qrow = query + (static_cast<int64_t>(s) * num_q_heads + kvh * G) * D;
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int k2 = 0; k2 < S::NCHUNK; ++k2) {
                const uint4 w = *reinterpret_cast<const uint4*>(qrow + g * D + k2 * 8 * S::LPT + 8 * c);
                qw[g][k2 * 4 + 0] = w.x;
                qw[g][k2 * 4 + 1] = w.y;
                qw[g][k2 * 4 + 2] = w.z;
                qw[g][k2 * 4 + 3] = w.w;
            }
        }
    }

    float m_run = -INFINITY;     // running max of head (lane % G), log2 units
    float l_run = 0.f;           // this lane's share of the running exp-sum
    float2 o2[G][EP];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < EP; ++e) o2[g][e] = make_float2(0.f, 0.f);

    bool aborted = false;
    int first_pending = 0;

    for (int k = 0; k < nk; ++k) {
        const int st = k % S::NSTAGE;
        if (!mbar_wait_bounded(&wbar[st], (k / S::NSTAGE) & 1)) {
            aborted = true;
            first_pending = k;
            break;
        }
        const int chunk = k >> 5;
        if (chunk != cons_chunk) {
            cons_tbl = load_table(chunk);
            cons_chunk = chunk;
        }
        const int phys = __shfl_sync(kFullMask, cons_tbl, k & 31);
        const bool ok = phys >= 0 && static_cast<int64_t>(phys) < num_blocks;
        const int nv = ok ? block_tokens(k) : 0;
        const unsigned char* stage = wstage + st * S::STAGE_BYTES;
#pragma unroll 1
        for (int tile = 0; tile < S::TILES; ++tile) {
            const unsigned char* ktile = stage + tile * S::CT * S::ROW_BYTES;
            const unsigned char* vtile = ktile + S::TILE_BYTES;
            const int tv = nv - tile * S::CT;     // valid tokens in this tile (may be <= 0)

            // ---- scores: this lane's partial dot products (fp32 accumulation) ----
            float acc[S::NVAL];
#pragma unroll
            for (int i = 0; i < S::NVAL; ++i) acc[i] = 0.f;
#pragma unroll
            for (int i = 0; i < S::ITERS; ++i) {
                const int t = i * S::RPW + r;
#pragma unroll
                for (int k2 = 0; k2 < S::NCHUNK; ++k2) {
                    const uint4 w = *reinterpret_cast<const uint4*>(
                        ktile + t * S::ROW_BYTES + (k2 * 8 * S::LPT + 8 * c) * 2);
                    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            acc[i * G + g] = fma_pair<T>(qw[g][k2 * 4 + j], words[j], acc[i * G + g]);
                }
            }
            const int base = transpose_reduce<S::NVAL, S::LPT>(acc, c);
#pragma unroll
            for (int j = 0; j < S::NHELD; ++j) {
                const int n = base + j;
                const int t = (n / G) * S::RPW + r;
                wscore[t * G + (n % G)] = t < tv ? acc[j] * scale_log2 : -INFINITY;
            }
            __syncwarp();

            // ---- blocked softmax, online: tile max, running max, rescale ----
            {
                const int g = lane % G;
                float sv[S::SM_TPL];
                float mloc = -INFINITY;
#pragma unroll
                for (int kk = 0; kk < S::SM_TPL; ++kk) {
                    const int t = lane / G + (32 / G) * kk;
                    sv[kk] = t < S::CT ? wscore[t * G + g] : -INFINITY;
                    mloc = fmaxf(mloc, sv[kk]);
                }
#pragma unroll
                for (int m = G; m < 32; m <<= 1) mloc = fmaxf(mloc, __shfl_xor_sync(kFullMask, mloc, m));
                const float m_new = fmaxf(m_run, mloc);
                const float m_sub = m_new == -INFINITY ? 0.f : m_new;
                const float corr = exp2f(m_run - m_sub);
                l_run *= corr;
#pragma unroll
                for (int kk = 0; kk < S::SM_TPL; ++kk) {
                    const int t = lane / G + (32 / G) * kk;
                    if (t < S::CT) {
                        const float p = exp2f(sv[kk] - m_sub);
                        l_run += p;
                        wscore[t * G + g] = p;
                    }
                }
                m_run = m_new;
                if (lane < G) wcorr[lane] = corr;
            }
            __syncwarp();

            // ---- values: rescale, then accumulate p * V (packed fp32 FMA) ----
            {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float cg = wcorr[g];
                    const float2 c2 = make_float2(cg, cg);
#pragma unroll
                    for (int e = 0; e < EP; ++e) o2[g][e] = __fmul2_rn(o2[g][e], c2);
                }
#pragma unroll
                for (int i = 0; i < S::ITERS; ++i) {
                    const int t = i * S::RPW + r;
                    if (t < tv) {
                        float2 p2[G];
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const float pg = wscore[t * G + g];
                            p2[g] = make_float2(pg, pg);
                        }
#pragma unroll
                        for (int k2 = 0; k2 < S::NCHUNK; ++k2) {
                            const uint4 w = *reinterpret_cast<const uint4*>(
                                vtile + t * S::ROW_BYTES + (k2 * 8 * S::LPT + 8 * c) * 2);
                            const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float2 vf = Elem<T>::to_float2(words[j]);
#pragma unroll
                                for (int g = 0; g < G; ++g)
                                    o2[g][k2 * 4 + j] = __ffma2_rn(p2[g], vf, o2[g][k2 * 4 + j]);
                            }
                        }
                    }
                }
            }
            __syncwarp();
        }
        if (issued < nk) issue(issued++);
    }

    if (aborted) {
        if (lane == 0) status_or(d_status, PA_STATUS_TIMEOUT);
        // Let the copies already started land (each wait bounded) before the
        // shared memory is reused.
        for (int k = first_pending; k < issued; ++k) {
            const int st = k % S::NSTAGE;
            mbar_wait_bounded(&wbar[st], (k / S::NSTAGE) & 1);
        }
    }

    // ---- merge inside the warp ----
#pragma unroll
    for (int m = G; m < 32; m <<= 1) l_run += __shfl_xor_sync(kFullMask, l_run, m);
#pragma unroll
    for (int m = S::LPT; m < 32; m <<= 1)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < EP; ++e) {
                o2[g][e].x += __shfl_xor_sync(kFullMask, o2[g][e].x, m);
                o2[g][e].y += __shfl_xor_sync(kFullMask, o2[g][e].y, m);
            }

    __syncthreads();   // every warp is done with its stage buffers
    float* epi_o = reinterpret_cast<float*>(smem);                 // [warp][g][D]
    float* epi_m = epi_o + kWarps * G * D;                         // [warp][g]
    float* epi_l = epi_m + kWarps * G;
    if (r == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k2 = 0; k2 < S::NCHUNK; ++k2) {
                float4* dst = reinterpret_cast<float4*>(epi_o + (warp * G + g) * D + k2 * 8 * S::LPT + 8 * c);
                dst[0] = make_float4(o2[g][k2 * 4 + 0].x, o2[g][k2 * 4 + 0].y,
                                     o2[g][k2 * 4 + 1].x, o2[g][k2 * 4 + 1].y);
                dst[1] = make_float4(o2[g][k2 * 4 + 2].x, o2[g][k2 * 4 + 2].y,
                                     o2[g][k2 * 4 + 3].x, o2[g][k2 * 4 + 3].y);
            }
    }
    if (lane < G) {
        epi_m[warp * G + lane] = m_run;
        epi_l[warp * G + lane] = l_run;
    }
    __syncthreads();

    merge_warps_and_store<T, D, G>(epi_o, epi_m, epi_l, out, ws_o, ws_ml, s, kvh, part, nparts,
                                   num_q_heads, max_parts);
}

}  // namespace pa

#include "paged_decode_mma.cuh"
#include "paged_decode_shared.cuh"
#include "paged_decode_q8.cuh"

namespace pa {

// One warp per (sequence, query head) whose context spans several
// partitions: merge the partitions' (max, exp-sum, normalised output).
template <typename T, int D>
__global__ void __launch_bounds__(kReduceRowsPerCta * 32) paged_decode_reduce_kernel(
    T* __restrict__ out, const float* __restrict__ ws_o, const float2* __restrict__ ws_ml,
    const int32_t* __restrict__ context_lens, int32_t num_seqs, int32_t num_q_heads,
    int32_t max_context_len, int32_t max_blocks_per_seq, int32_t block_size,
    int32_t partition_size, int32_t max_parts)
{
    grid_dependency_wait();
    constexpr int EPL = D / 32;     // elements per lane
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kReduceRowsPerCta + (threadIdx.x >> 5);
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
    for (int p = 0; p < np; ++p) {
        const float2 v = ml[p];
        const float w = v.y * exp2f(v.x - msub);
        W += w;
        if (EPL == 4) {
            const float4 x = *reinterpret_cast<const float4*>(orow + static_cast<int64_t>(p) * D);
            acc[0] = fmaf(w, x.x, acc[0]);
            acc[1] = fmaf(w, x.y, acc[1]);
            acc[2] = fmaf(w, x.z, acc[2]);
            acc[3] = fmaf(w, x.w, acc[3]);
        } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, orow[static_cast<int64_t>(p) * D + e], acc[e]);
        }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    T* dst = out + row * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
        const uint32_t packed = Elem<T>::from_float2(acc[e] * inv, acc[e + 1] * inv);
        *reinterpret_cast<uint32_t*>(dst + e) = packed;
    }
}

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
// box is one block of one kv head: B rows of D bytes, with the 128-byte
// swizzle when a row is 128 bytes (else dense).
static bool encode_pool_map_q8(CUtensorMap* map, const void* pool, int32_t head_dim,
                                int32_t num_kv_heads, int32_t block_size, int64_t num_blocks)
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
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(head_dim), 1u,
                               static_cast<cuuint32_t>(block_size), 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult res = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(pool), dims,
                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS;
}

template <typename Codes, typename T, int D, int BS, int G>
static pa_status launch_decode_q8(const DecodeArgs& a, float v_scale)
{
    using S = Q8Shape<D, BS, G>;
    static std::atomic<uint64_t> attr_done{0};
    auto kernel = std::is_same<Codes, Int8Codes>::value ? paged_decode_int8_kernel<T, D, BS, G>
                                                        : paged_decode_fp8_kernel<T, D, BS, G>;
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
        static_cast<uint8_t*>(const_cast<void*>(a.v_cache)), a.num_kv_heads, a.k_inv, a.v_inv);
    if (st != PA_OK || a.max_parts <= 1) return st;
    const int64_t rows = static_cast<int64_t>(a.num_seqs) * a.num_q_heads;
    const unsigned ctas = static_cast<unsigned>((rows + kReduceRowsPerCta - 1) / kReduceRowsPerCta);
    return launch_overlapped(paged_decode_reduce_kernel<T, D>, dim3(ctas),
                             dim3(kReduceRowsPerCta * 32), 0, a.stream, static_cast<T*>(a.out),
                             a.ws_o, a.ws_ml, a.context_lens, a.num_seqs, a.num_q_heads,
                             a.max_context_len, a.max_blocks_per_seq, a.block_size,
                             a.partition_size, a.max_parts);
}

template <typename Codes, typename T, int D, int BS>
static pa_status dispatch_q8_group(const DecodeArgs& a, float v_scale)
{
    switch (a.num_q_heads / a.num_kv_heads) {
    case 1: return launch_decode_q8<Codes, T, D, BS, 1>(a, v_scale);
    case 2: return launch_decode_q8<Codes, T, D, BS, 2>(a, v_scale);
    case 4: return launch_decode_q8<Codes, T, D, BS, 4>(a, v_scale);
    case 8: return launch_decode_q8<Codes, T, D, BS, 8>(a, v_scale);
    default: return PA_ERR_UNSUPPORTED;
    }
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
            a.num_kv_heads, a.lpt_seqs);
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
            a.num_kv_heads, a.lpt_seqs);
        if (ls != PA_OK) return ls;
    }
    if (a.max_parts <= 1) return PA_OK;
    const int64_t rows = static_cast<int64_t>(a.num_seqs) * a.num_q_heads;
    const unsigned ctas = static_cast<unsigned>((rows + kReduceRowsPerCta - 1) / kReduceRowsPerCta);
    return launch_overlapped(paged_decode_reduce_kernel<T, D>, dim3(ctas),
                             dim3(kReduceRowsPerCta * 32), 0, a.stream, static_cast<T*>(a.out),
                             a.ws_o, a.ws_ml, a.context_lens, a.num_seqs, a.num_q_heads,
                             a.max_context_len, a.max_blocks_per_seq, a.block_size,
                             a.partition_size, a.max_parts);
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
        a.max_parts, a.ws_o, a.ws_ml, a.d_status);
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
                             float v_scale = 1.f)
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

extern "C" pa_status pa_paged_decode_shared_prefix(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, const int32_t* prefix_lens,
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
    int32_t max_context_len, int32_t max_prefix_len, float scale, int32_t partition_size,
    void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* d_status, pa_stream_t stream)
{
    using namespace pa;
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
    return dtype == PA_DTYPE_F16 ? dispatch_shared<__half>(sa) : dispatch_shared<__nv_bfloat16>(sa);
}

// ---------------------------------------------------------------------------
// pa_paged_decode_no_alloc: the same decode with its split-context scratch in
// a file-scope device array instead of caller memory.
// ---------------------------------------------------------------------------
namespace pa {

static __device__ __align__(256) unsigned char g_no_alloc_workspace[PA_NO_ALLOC_WORKSPACE_BYTES];

static std::mutex g_no_alloc_mutex;
static void* g_no_alloc_ptr[kMaxDevices];   // device address of the array, per device

// Device address of the array on the current device; looked up once per
// device (host code may not use the symbol itself as a device pointer).
static pa_status no_alloc_workspace(void** ptr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_no_alloc_mutex);
    if (g_no_alloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_no_alloc_workspace) != cudaSuccess || p == nullptr)
            return PA_ERR_CUDA;
        g_no_alloc_ptr[dev] = p;
    }
    *ptr = g_no_alloc_ptr[dev];
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
