// paged_decode_mma.cuh -- the decode kernel for grouped query heads (G >= 4)
// with warp-level tensor-core contractions.  Included by paged_decode.cu.
//
// Same work split, pipeline and softmax as paged_decode_kernel: one CTA per
// (kv head, context partition, sequence), four warps each streaming every
// fourth physical block of the partition through a shared-memory ring filled
// by TMA, the blocked softmax of "PagedAttention：大模型KV Cache分页管理优化实践"
// §5.1 run online, and the same fixed-order merge.  What differs is how a
// block's tokens meet the G query heads of the kv head: a block of 16 tokens
// times G heads is a dense 16 x 128 x G contraction for q.k and again for
// p.V, so each is done with mma.sync m16n8k16 (16-bit inputs, fp32
// accumulation) instead of per-lane fp32 FMAs, which cut the instructions
// per byte enough for the kernel to stay bandwidth-bound.
//
// Layout of the contractions (one warp, one 16-token slice of a block):
//   S[g][t] = sum_d q[g][d] K[t][d]:  A = q (rows = heads, rows >= G are
//     zero), B = K^T read with ldmatrix from the K tile, C = S in fp32;
//   O[g][d] += sum_t P[g][t] V[t][d]: A = P, taken straight from the S
//     accumulator registers after the softmax (rounded to the input type),
//     B = V read with ldmatrix.trans from the V tile.
// K and V tiles land in shared memory through a 5-D tensor map with the
// 128-byte swizzle: row r (one token's 64 dims, 128 bytes) keeps its 16-byte
// chunk c at chunk c ^ (r % 8), so the 8 rows an ldmatrix reads fall in
// different banks.
#pragma once

#include "decode_common.cuh"

namespace pa {

template <int D, int BS, int G>
struct MmaShape {
    static constexpr int NH = D / 64;                 // 128-byte halves of a token row
    static constexpr int KSTEPS = D / 16;             // k-steps of q.k
    static constexpr int NTILES = D / 8;              // 8-wide n-tiles of the output
    static constexpr int SLICES = BS / 16;            // 16-token slices per block
    static constexpr int TILE_BYTES = BS * D * 2;     // K (or V) of one block, one head
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int NSTAGE = 2;
    static constexpr int WARP_STAGE_BYTES = NSTAGE * STAGE_BYTES;
    static constexpr int OFF_BARS = kWarps * WARP_STAGE_BYTES;
    // + a probe barrier per warp, + alignment slack
    static constexpr int SMEM_BYTES = OFF_BARS + kWarps * (NSTAGE + 1) * 8 + 1024;
    static constexpr int EPI_BYTES = kWarps * G * (D + 2) * 4;
    static_assert(BS % 16 == 0, "whole 16-token slices");
    static_assert(D % 64 == 0, "whole 128-byte rows");
    static_assert(G >= 2 && G <= 8, "heads fit the 16 rows of the A operand");
    static_assert(EPI_BYTES <= OFF_BARS, "epilogue fits in the stage buffers");
    static_assert(TILE_BYTES % 1024 == 0, "tiles keep the 1024-byte swizzle alignment");
};

// Byte offset, inside a swizzled tile, of the 16-byte chunk holding elements
// [8 * chunk, 8 * chunk + 8) of token t: row = half * BS + t.
template <int BS>
__device__ __forceinline__ uint32_t swz_offset(int t, int dim)
{
    const int row = (dim >> 6) * BS + t;
    const int c = (dim >> 3) & 7;
    return static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4));
}

template <typename T>
__device__ __forceinline__ uint32_t pack_pair(float lo, float hi)
{
    return Elem<T>::from_float2(lo, hi);
}

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(kThreads, 3) paged_decode_mma_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    T* __restrict__ out, const T* __restrict__ query, const int32_t* __restrict__ block_tables,
    const int32_t* __restrict__ context_lens, int32_t num_q_heads, int32_t max_blocks_per_seq,
    int64_t num_blocks, int32_t max_context_len, float scale_log2, int32_t partition_size,
    int32_t max_parts, float* __restrict__ ws_o, float2* __restrict__ ws_ml, int32_t* d_status,
    const T* __restrict__ new_key, const T* __restrict__ new_value, T* __restrict__ k_cache,
    T* __restrict__ v_cache, int32_t num_kv_heads, int32_t lpt_seqs, uint32_t probe_us)
{
    grid_dependency_wait();   // before any global access (see pa_common.cuh)
    using S = MmaShape<D, BS, G>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // the 128-byte swizzle repeats every 1024 bytes: align the tiles to it
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int kvh = blockIdx.x;
    const int part = blockIdx.y;
    const int s = lpt_seqs > 0
                      ? lpt_sequence(context_lens, block_tables, max_blocks_per_seq, lpt_seqs,
                                     blockIdx.z, reinterpret_cast<int32_t*>(smem))
                      : static_cast<int>(blockIdx.z);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int grp = lane >> 2;          // row group of the mma fragments (head)
    const int tig = lane & 3;           // thread in group (column pair)

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
    const int nk = warp < nblk ? (nblk - warp + kWarps - 1) / kWarps : 0;
    const int append_blk = (new_key != nullptr && part == nparts - 1) ? (ctx - 1) / BS - blk_begin : -1;

    unsigned char* wstage = smem + warp * S::WARP_STAGE_BYTES;
    uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + S::OFF_BARS) + warp * (S::NSTAGE + 1);

    if (lane == 0) {
#pragma unroll
        for (int st = 0; st <= S::NSTAGE; ++st) mbar_init(&wbar[st], 1);   // + the probe barrier
        fence_barrier_init();
    }
    __syncwarp();

    const int32_t* table = block_tables + static_cast<int64_t>(s) * max_blocks_per_seq + blk_begin;
    auto load_table = [&](int chunk) -> int {
        const int kk = chunk * 32 + lane;
        return kk < nk ? table[warp + kWarps * kk] : -1;
    };
    int prod_chunk = 0, cons_chunk = 0;
    int prod_tbl = lane < nk ? pre_tbl : -1;   // load_table(0), already in flight
    int cons_tbl = prod_tbl;

    auto block_tokens = [&](int k) -> int {
        const int t0 = tok_begin + (warp + kWarps * k) * BS;
        return min(BS, tok_end - t0);
    };

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
                tma_load_5d(dst, &tm_k, 0, 0, 0, kvh, phys, &wbar[st]);
                tma_load_5d(dst + S::TILE_BYTES, &tm_v, 0, 0, 0, kvh, phys, &wbar[st]);
            } else {
                status_or(d_status, PA_STATUS_BAD_BLOCK);
                mbar_arrive_expect_tx(&wbar[st], 0u);
            }
        }
    };

    const int prologue = min(nk, S::NSTAGE);
    for (int k = 0; k < prologue; ++k) issue(k);
    int issued = prologue;

    // A fragments of q (rows = heads): for k-step ks, lane holds
    // q[grp][16 ks + 2 tig .. +1] and q[grp][16 ks + 8 + 2 tig .. +1];
    // rows 8..15 of A are zero, as are rows grp >= G.
    uint32_t qa[S::KSTEPS][2];
    {
        const T* qrow = query + (static_cast<int64_t>(s) * num_q_heads + kvh * G + grp) * D;
#pragma unroll
        for (int ks = 0; ks < S::KSTEPS; ++ks) {
            qa[ks][0] = grp < G ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * tig) : 0u;
            qa[ks][1] = grp < G ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * tig) : 0u;
        }
    }

    // ldmatrix lane roles: lane gives row (lane % 8) of matrix (lane / 8)
    const int mi = lane >> 3;
    const int ri = lane & 7;

    float m_run = -INFINITY;     // running max of head grp (log2 units)
    float l_run = 0.f;           // this lane's share of head grp's exp-sum
    float o[S::NTILES][4];       // O[grp][8 nt + 2 tig .. +1] in [0..1]; rows 8..15 in [2..3]
#pragma unroll
    for (int nt = 0; nt < S::NTILES; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;

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
        unsigned char* ktile = wstage + st * S::STAGE_BYTES;
        unsigned char* vtile = ktile + S::TILE_BYTES;
        const uint32_t ks_base = smem_u32(ktile);
        const uint32_t vs_base = smem_u32(vtile);

        if (nv < BS) {
            // Rows past the context (or of a block that was not loaded) may
            // hold anything, NaN included; p = 0 does not cancel a NaN in
            // the tensor-core sum, so clear those V rows.
            const int lines = (BS - nv) * S::NH * 8;          // 16-byte chunks
            for (int i = lane; i < lines; i += 32) {
                const int chunk16 = i & 7;
                const int rowi = i >> 3;                        // (token, half) pairs
                const int t = nv + rowi / S::NH;
                const int h = rowi % S::NH;
                *reinterpret_cast<uint4*>(vtile + (h * BS + t) * 128 + chunk16 * 16) =
                    make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }

#pragma unroll 1
        for (int sl = 0; sl < S::SLICES; ++sl) {
            const int t0 = sl * 16;
            const int tv = nv - t0;         // valid tokens in this slice (may be <= 0)

            // ---- S = q K^T for 16 tokens (two 8-token n-tiles) ----
            float sc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
                const int t = t0 + nt * 8 + ri;
#pragma unroll
                for (int kp = 0; kp < S::KSTEPS / 2; ++kp) {
                    uint32_t b[4];
                    ldmatrix_x4(b, ks_base + swz_offset<BS>(t, kp * 32 + mi * 8));
                    mma_16816<T>(sc[nt], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, b[0], b[1]);
                    mma_16816<T>(sc[nt], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, b[2], b[3]);
                }
            }

            // ---- blocked softmax, online, for head grp ----
            // lane holds tokens t0 + 2 tig, +1 (n-tile 0) and t0 + 8 + 2 tig, +1 (n-tile 1)
            float x[4];
            x[0] = 2 * tig < tv ? sc[0][0] * scale_log2 : -INFINITY;
            x[1] = 2 * tig + 1 < tv ? sc[0][1] * scale_log2 : -INFINITY;
            x[2] = 8 + 2 * tig < tv ? sc[1][0] * scale_log2 : -INFINITY;
            x[3] = 8 + 2 * tig + 1 < tv ? sc[1][1] * scale_log2 : -INFINITY;
            float mloc = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
            mloc = fmaxf(mloc, __shfl_xor_sync(kFullMask, mloc, 1));
            mloc = fmaxf(mloc, __shfl_xor_sync(kFullMask, mloc, 2));
            const float m_new = fmaxf(m_run, mloc);
            const float m_sub = m_new == -INFINITY ? 0.f : m_new;
            const float corr = exp2f(m_run - m_sub);
            m_run = m_new;
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) p[e] = grp < G ? exp2f(x[e] - m_sub) : 0.f;
            // P as the A operand, in the input type; the exp-sum adds the
            // rounded values so that the weights sum exactly to it.
            const uint32_t pa0 = pack_pair<T>(p[0], p[1]);
            const uint32_t pa2 = pack_pair<T>(p[2], p[3]);
            const float2 r0 = Elem<T>::to_float2(pa0), r2 = Elem<T>::to_float2(pa2);
            l_run = l_run * corr + ((r0.x + r0.y) + (r2.x + r2.y));
#pragma unroll
            for (int nt = 0; nt < S::NTILES; ++nt) {
                o[nt][0] *= corr;
                o[nt][1] *= corr;
            }

            // ---- O += P V for 16 tokens ----
            {
                const int t = t0 + (mi & 1) * 8 + ri;
#pragma unroll
                for (int np = 0; np < S::NTILES / 2; ++np) {
                    uint32_t b[4];
                    ldmatrix_x4_trans(b, vs_base + swz_offset<BS>(t, np * 16 + (mi >> 1) * 8));
                    mma_16816<T>(o[2 * np], pa0, 0u, pa2, 0u, b[0], b[1]);
                    mma_16816<T>(o[2 * np + 1], pa0, 0u, pa2, 0u, b[2], b[3]);
                }
            }
        }
        __syncwarp();
        if (issued < nk) issue(issued++);
    }

    if (aborted) drain_after_timeout<S::NSTAGE>(wbar, first_pending, issued, d_status);

    // ---- merge inside the warp: exp-sum across the 4 lanes of a head ----
    l_run += __shfl_xor_sync(kFullMask, l_run, 1);
    l_run += __shfl_xor_sync(kFullMask, l_run, 2);

    // every warp is done with its stage buffers, unless one gave up waiting
    if (__syncthreads_or(aborted)) {
        store_aborted_rows<T, D, G>(out, ws_o, ws_ml, s, kvh, part, nparts, num_q_heads, max_parts);
        return;
    }
    float* epi_o = reinterpret_cast<float*>(smem);                 // [warp][g][D]
    float* epi_m = epi_o + kWarps * G * D;                         // [warp][g]
    float* epi_l = epi_m + kWarps * G;
    if (grp < G) {
#pragma unroll
        for (int nt = 0; nt < S::NTILES; ++nt)
            *reinterpret_cast<float2*>(epi_o + (warp * G + grp) * D + nt * 8 + 2 * tig) =
                make_float2(o[nt][0], o[nt][1]);
        if (tig == 0) {
            epi_m[warp * G + grp] = m_run;
            epi_l[warp * G + grp] = l_run;
        }
    }
    __syncthreads();
    merge_warps_and_store<T, D, G>(epi_o, epi_m, epi_l, out, ws_o, ws_ml, s, kvh, part, nparts,
                                   num_q_heads, max_parts);
}

}  // namespace pa
