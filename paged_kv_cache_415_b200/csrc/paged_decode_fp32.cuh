// paged_decode_fp32.cuh -- the decode kernel for query groups G < 4 with
// fp32 CUDA-core arithmetic.  Included by paged_decode.cu.
//
// paged_decode_kernel: one CTA per (kv head, context partition, sequence).
// The CTA carries the G = Hq / Hkv query heads of its kv head, so every K/V
// byte is read from HBM once for all of them.  Each of its four warps runs
// its own pipeline over every fourth physical block of the partition:
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
#pragma once

#include "decode_common.cuh"

namespace pa {

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
    static constexpr int SMEM_BYTES = OFF_BARS + kWarps * (NSTAGE + 1) * 8;   // + a probe barrier
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

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(kThreads, (DecodeShape<D, BS, G>::MIN_CTAS)) paged_decode_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    T* __restrict__ out, const T* __restrict__ query, const int32_t* __restrict__ block_tables,
    const int32_t* __restrict__ context_lens, int32_t num_q_heads, int32_t max_blocks_per_seq,
    int64_t num_blocks, int32_t max_context_len, float scale_log2, int32_t partition_size,
    int32_t max_parts, float* __restrict__ ws_o, float2* __restrict__ ws_ml, int32_t* d_status,
    const T* __restrict__ new_key, const T* __restrict__ new_value, T* __restrict__ k_cache,
    T* __restrict__ v_cache, int32_t num_kv_heads, int32_t lpt_seqs, uint32_t probe_us)
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
    uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + S::OFF_BARS) + warp * (S::NSTAGE + 1);

    if (lane == 0) {
#pragma unroll
        for (int st = 0; st <= S::NSTAGE; ++st) mbar_init(&wbar[st], 1);   // + the probe barrier
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

    bool aborted = nk > 0 && probe_gives_up(&wbar[S::NSTAGE], probe_us);
    int first_pending = 0;

    for (int k = 0; k < (aborted ? 0 : nk); ++k) {
        const int st = k % S::NSTAGE;
        if (!mbar_wait_warp(&wbar[st], (k / S::NSTAGE) & 1)) {
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

    if (aborted) drain_after_timeout<S::NSTAGE>(wbar, first_pending, issued, d_status);

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

    // every warp is done with its stage buffers, unless one gave up waiting
    if (__syncthreads_or(aborted)) {
        store_aborted_rows<T, D, G>(out, ws_o, ws_ml, s, kvh, part, nparts, num_q_heads, max_parts);
        return;
    }
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
