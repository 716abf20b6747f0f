// paged_decode_shared.cuh -- decode for batches whose sequences come in
// groups that share a stored prefix (the beams of one prompt, parallel
// samples of one request).  Included by paged_decode.cu.
//
// "PagedAttention：大模型KV Cache分页管理优化实践" §5.2 (非连续KV访问优化), step 1:
// process together the queries that touch the same physical block.  With
// block sharing ("vLLM用虚拟内存分页思想管理KV Cache", 写时复制与块共享机制) the
// members of a group point at the same physical blocks for their first
// prefix_len tokens, so those blocks are read from HBM once for the whole
// group: the members' query heads become extra rows of the tensor-core
// tile, exactly as the query heads of a GQA group do.
//
// A work item is (kv head, part, group z).  The group's blocks form one list:
// the prefix blocks [0, L / B) through the first member's table (every
// member's rows of the tile live: rows = members x G <= 8), then each
// member's private blocks [L / B, ceil(ctx / B)) in member order (only that
// member's G rows live; the others' scores are masked out).  The list is
// cut into parts of part_blocks blocks; a part's blocks are dealt
// round-robin to the four warps.  A group whose list fits one part writes
// its output rows directly; otherwise each part leaves (max, exp-sum,
// normalised output) partials that a reduction merges with the rule of
// §5.1.  So a private suffix costs no CTA of its own and no merge.
#pragma once

#include "decode_common.cuh"
#include "paged_decode_mma.cuh"   // swz_offset, pack_pair

namespace pa {

constexpr int kSharedRows = 8;   // query rows per tile (rows 0..7 of the A operand)

template <int D, int BS>
struct SharedShape {
    static constexpr int NH = D / 64;
    static constexpr int KSTEPS = D / 16;
    static constexpr int NTILES = D / 8;
    static constexpr int SLICES = BS / 16;
    static constexpr int TILE_BYTES = BS * D * 2;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int NSTAGE = 2;
    static constexpr int WARP_STAGE_BYTES = NSTAGE * STAGE_BYTES;
    static constexpr int OFF_BARS = kWarps * WARP_STAGE_BYTES;
    // + a probe barrier per warp, + alignment slack
    static constexpr int SMEM_BYTES = OFF_BARS + kWarps * (NSTAGE + 1) * 8 + 1024;
    static constexpr int EPI_BYTES = kWarps * kSharedRows * (D + 2) * 4;
    static_assert(BS % 16 == 0 && D % 64 == 0, "whole 16-token slices, 128-byte rows");
    static_assert(EPI_BYTES <= OFF_BARS, "epilogue fits in the stage buffers");
    static_assert(TILE_BYTES % 1024 == 0, "tiles keep the 1024-byte swizzle alignment");
};

// Whether group z's prefix is usable: a whole number of blocks, within the
// caller's bound, and no longer than any member's (valid) context.  The
// prefix work items and the reduction evaluate it the same way.
__device__ __forceinline__ bool prefix_ok(const int32_t* context_lens, int32_t L, int z,
                                          int group_size, int block_size, int32_t max_prefix_len,
                                          int32_t max_context_len, int32_t max_tokens)
{
    if (L < 0 || L % block_size != 0 || L > max_prefix_len) return false;
    for (int j = 0; j < group_size; ++j) {
        const int32_t c = context_lens[z * group_size + j];
        if (c < 0 || c > max_context_len || c > max_tokens || c < L) return false;
    }
    return true;
}

// Group z's list of blocks: the shared prefix, then each member's own.
__device__ __forceinline__ int group_blocks(const int32_t* __restrict__ context_lens, int seq0,
                                            int group_size, int nb_pre, int block_size)
{
    int total = nb_pre;
    for (int j = 0; j < group_size; ++j)
        total += (context_lens[seq0 + j] + block_size - 1) / block_size - nb_pre;
    return total;
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads, 3) paged_decode_shared_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    T* __restrict__ out, const T* __restrict__ query, const int32_t* __restrict__ block_tables,
    const int32_t* __restrict__ context_lens, const int32_t* __restrict__ prefix_lens,
    int32_t group_size, int32_t G, int32_t num_q_heads, int32_t max_blocks_per_seq,
    int64_t num_blocks, int32_t max_context_len, int32_t max_prefix_len, float scale_log2,
    int32_t part_blocks, int32_t max_parts, float* __restrict__ ws_o, float2* __restrict__ ws_ml,
    int32_t* d_status, uint32_t probe_us)
{
    grid_dependency_wait();   // before any global access (see pa_common.cuh)
    using S = SharedShape<D, BS>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int kvh = blockIdx.x;
    const int part = blockIdx.y;
    const int z = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int grp = lane >> 2;
    const int tig = lane & 3;
    const int32_t max_tokens = max_blocks_per_seq * BS;
    const int seq0 = z * group_size;
    const int rows = group_size * G;

    // output rows of the group for this kv head, all zero
    auto zero_rows = [&]() {
        for (int idx = threadIdx.x; idx < rows * (D / 8); idx += kThreads) {
            const int r = idx / (D / 8);
            const int64_t row = static_cast<int64_t>(seq0 + r / G) * num_q_heads + kvh * G + r % G;
            reinterpret_cast<uint4*>(out + row * D)[idx % (D / 8)] = make_uint4(0, 0, 0, 0);
        }
    };
    const int32_t L = prefix_lens[z];
    if (!prefix_ok(context_lens, L, z, group_size, BS, max_prefix_len, max_context_len,
                   max_tokens)) {
        if (part == 0) {
            zero_rows();
            if (threadIdx.x == 0) status_or(d_status, PA_STATUS_BAD_CONTEXT);
        }
        return;
    }
    const int nb_pre = L / BS;
    const int total = group_blocks(context_lens, seq0, group_size, nb_pre, BS);
    if (total == 0) {                        // every member's context is empty
        if (part == 0) zero_rows();
        return;
    }
    const int nparts = (total + part_blocks - 1) / part_blocks;
    const int v_begin = part * part_blocks;
    if (v_begin >= total) return;
    const int nblk = min(part_blocks, total - v_begin);
    const int nk = warp < nblk ? (nblk - warp + kWarps - 1) / kWarps : 0;

    unsigned char* wstage = smem + warp * S::WARP_STAGE_BYTES;
    uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + S::OFF_BARS) + warp * (S::NSTAGE + 1);
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st <= S::NSTAGE; ++st) mbar_init(&wbar[st], 1);   // + the probe barrier
        fence_barrier_init();
    }
    __syncwarp();

    // Block v of the list: its physical id and (valid tokens | (member + 1)
    // << 8), member -1 for a shared prefix block.  Every member's entry for
    // a prefix block must name the same physical block.
    auto resolve = [&](int v, int& phys, int& info) {
        if (v < nb_pre) {
            const int32_t e = block_tables[static_cast<int64_t>(seq0) * max_blocks_per_seq + v];
            bool same = true;
            for (int m = 1; m < group_size; ++m)
                same &= block_tables[static_cast<int64_t>(seq0 + m) * max_blocks_per_seq + v] == e;
            if (!same) status_or(d_status, PA_STATUS_BAD_BLOCK);
            phys = e;
            info = BS;
            return;
        }
        int r = v - nb_pre;
        for (int j = 0; j < group_size; ++j) {
            const int32_t c = context_lens[seq0 + j];
            const int n = (c + BS - 1) / BS - nb_pre;
            if (r < n) {
                const int b = nb_pre + r;
                phys = block_tables[static_cast<int64_t>(seq0 + j) * max_blocks_per_seq + b];
                info = min(BS, c - b * BS) | ((j + 1) << 8);
                return;
            }
            r -= n;
        }
        phys = -1;
        info = 0;
    };
    // one list entry per lane, 32 blocks of this warp per load
    auto load_chunk = [&](int chunk, int& phys, int& info) {
        const int kk = chunk * 32 + lane;
        phys = -1;
        info = 0;
        if (kk < nk) resolve(v_begin + warp + kWarps * kk, phys, info);
    };
    int prod_chunk = 0, cons_chunk = 0;
    int prod_phys, prod_info;
    load_chunk(0, prod_phys, prod_info);
    int cons_phys = prod_phys, cons_info = prod_info;

    auto issue = [&](int k) {
        const int chunk = k >> 5;
        if (chunk != prod_chunk) {
            load_chunk(chunk, prod_phys, prod_info);
            prod_chunk = chunk;
        }
        const int phys = __shfl_sync(kFullMask, prod_phys, k & 31);
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

    // Row grp of the A operand: member grp / G's query head kvh * G + grp % G.
    const bool row_live = grp < rows;
    const int row_member = row_live ? grp / G : -2;
    uint32_t qa[S::KSTEPS][2];
    {
        const int member = row_live ? grp / G : 0;
        const int h = kvh * G + (row_live ? grp % G : 0);
        const T* qrow = query + (static_cast<int64_t>(seq0 + member) * num_q_heads + h) * D;
#pragma unroll
        for (int ks = 0; ks < S::KSTEPS; ++ks) {
            qa[ks][0] = row_live ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * tig) : 0u;
            qa[ks][1] = row_live ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * tig) : 0u;
        }
    }

    const int mi = lane >> 3;
    const int ri = lane & 7;
    float m_run = -INFINITY;
    float l_run = 0.f;
    float o[S::NTILES][4];
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
            load_chunk(chunk, cons_phys, cons_info);
            cons_chunk = chunk;
        }
        const int phys = __shfl_sync(kFullMask, cons_phys, k & 31);
        const int info = __shfl_sync(kFullMask, cons_info, k & 31);
        const bool ok = phys >= 0 && static_cast<int64_t>(phys) < num_blocks;
        const int nv = ok ? (info & 0xff) : 0;
        const int owner = (info >> 8) - 1;            // -1: shared by every member
        // this lane's row takes part in this block's scores
        const bool row_on = row_live && (owner < 0 || owner == row_member);
        unsigned char* ktile = wstage + st * S::STAGE_BYTES;
        unsigned char* vtile = ktile + S::TILE_BYTES;
        const uint32_t ks_base = smem_u32(ktile);
        const uint32_t vs_base = smem_u32(vtile);

        if (nv < BS) {                      // clear V rows that may hold anything
            const int lines = (BS - nv) * S::NH * 8;
            for (int i = lane; i < lines; i += 32) {
                const int rowi = i >> 3;
                const int t = nv + rowi / S::NH;
                const int h = rowi % S::NH;
                *reinterpret_cast<uint4*>(vtile + (h * BS + t) * 128 + (i & 7) * 16) =
                    make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }

#pragma unroll 1
        for (int sl = 0; sl < S::SLICES; ++sl) {
            const int t0 = sl * 16;
            const int tv = row_on ? nv - t0 : 0;     // tokens this row may see
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
            for (int e = 0; e < 4; ++e) p[e] = row_live ? exp2f(x[e] - m_sub) : 0.f;
            const uint32_t pa0 = pack_pair<T>(p[0], p[1]);
            const uint32_t pa2 = pack_pair<T>(p[2], p[3]);
            const float2 r0 = Elem<T>::to_float2(pa0), r2 = Elem<T>::to_float2(pa2);
            l_run = l_run * corr + ((r0.x + r0.y) + (r2.x + r2.y));
#pragma unroll
            for (int nt = 0; nt < S::NTILES; ++nt) {
                o[nt][0] *= corr;
                o[nt][1] *= corr;
            }
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

    l_run += __shfl_xor_sync(kFullMask, l_run, 1);
    l_run += __shfl_xor_sync(kFullMask, l_run, 2);

    // every warp is done with its stage buffers, unless one gave up waiting:
    // then the group's rows get "nothing" through global memory only (zero
    // rows, or an empty partial the reduction weighs with 0)
    if (__syncthreads_or(aborted)) {
        for (int idx = threadIdx.x; idx < rows * (D / 8); idx += kThreads) {
            const int r = idx / (D / 8);
            const int d0 = (idx % (D / 8)) * 8;
            const int64_t row = static_cast<int64_t>(seq0 + r / G) * num_q_heads + kvh * G + r % G;
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
        return;
    }
    float* epi_o = reinterpret_cast<float*>(smem);                    // [warp][row][D]
    float* epi_m = epi_o + kWarps * kSharedRows * D;                  // [warp][row]
    float* epi_l = epi_m + kWarps * kSharedRows;
    if (row_live) {
#pragma unroll
        for (int nt = 0; nt < S::NTILES; ++nt)
            *reinterpret_cast<float2*>(epi_o + (warp * kSharedRows + grp) * D + nt * 8 + 2 * tig) =
                make_float2(o[nt][0], o[nt][1]);
        if (tig == 0) {
            epi_m[warp * kSharedRows + grp] = m_run;
            epi_l[warp * kSharedRows + grp] = l_run;
        }
    }
    __syncthreads();

    // merge the warps in a fixed order: the output row, or this part's partial
    for (int idx = threadIdx.x; idx < rows * (D / 8); idx += kThreads) {
        const int r = idx / (D / 8);
        const int d0 = (idx % (D / 8)) * 8;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, epi_m[w * kSharedRows + r]);
        const float msub = M == -INFINITY ? 0.f : M;
        float Lsum = 0.f;
        float O[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) O[e] = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float f = exp2f(epi_m[w * kSharedRows + r] - msub);
            Lsum = fmaf(f, epi_l[w * kSharedRows + r], Lsum);
            const float4* src = reinterpret_cast<const float4*>(epi_o + (w * kSharedRows + r) * D + d0);
            const float4 a = src[0], b = src[1];
            O[0] = fmaf(f, a.x, O[0]); O[1] = fmaf(f, a.y, O[1]);
            O[2] = fmaf(f, a.z, O[2]); O[3] = fmaf(f, a.w, O[3]);
            O[4] = fmaf(f, b.x, O[4]); O[5] = fmaf(f, b.y, O[5]);
            O[6] = fmaf(f, b.z, O[6]); O[7] = fmaf(f, b.w, O[7]);
        }
        const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) O[e] *= inv;
        const int64_t row = static_cast<int64_t>(seq0 + r / G) * num_q_heads + kvh * G + r % G;
        if (nparts == 1) {
            *reinterpret_cast<uint4*>(out + row * D + d0) = pack8<T>(O);
        } else {
            const int64_t prow = row * max_parts + part;
            float4* dst = reinterpret_cast<float4*>(ws_o + prow * D + d0);
            dst[0] = make_float4(O[0], O[1], O[2], O[3]);
            dst[1] = make_float4(O[4], O[5], O[6], O[7]);
            if (d0 == 0) ws_ml[prow] = make_float2(M, Lsum);
        }
    }
}

// One warp per (sequence, query head) of a group whose block list spans
// several parts: merge the parts' partials into the output row.  Groups that
// fit one part (or were refused) were written by the decode kernel.
template <typename T, int D>
__global__ void __launch_bounds__(kReduceRowsPerCta * 32) paged_decode_shared_reduce_kernel(
    T* __restrict__ out, const float* __restrict__ ws_o, const float2* __restrict__ ws_ml,
    const int32_t* __restrict__ context_lens, const int32_t* __restrict__ prefix_lens,
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t max_context_len,
    int32_t max_blocks_per_seq, int32_t block_size, int32_t max_prefix_len, int32_t part_blocks,
    int32_t max_parts)
{
    grid_dependency_wait();
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kReduceRowsPerCta + (threadIdx.x >> 5);
    if (row >= static_cast<int64_t>(num_seqs) * num_q_heads) return;
    const int s = static_cast<int>(row / num_q_heads);
    const int z = s / group_size;
    const int32_t L = prefix_lens[z];
    if (!prefix_ok(context_lens, L, z, group_size, block_size, max_prefix_len, max_context_len,
                   max_blocks_per_seq * block_size))
        return;
    const int total = group_blocks(context_lens, z * group_size, group_size, L / block_size,
                                   block_size);
    const int n = (total + part_blocks - 1) / part_blocks;
    if (n <= 1) return;
    const float2* ml = ws_ml + row * max_parts;
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) M = fmaxf(M, ml[i].x);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, m));
    const float msub = M == -INFINITY ? 0.f : M;
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    float W = 0.f;
    const float* orow = ws_o + row * max_parts * D + lane * EPL;
    for (int i = 0; i < n; ++i) {
        const float2 v = ml[i];
        const float w = v.y * exp2f(v.x - msub);
        W += w;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, orow[static_cast<int64_t>(i) * D + e], acc[e]);
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    T* dst = out + row * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; e += 2)
        *reinterpret_cast<uint32_t*>(dst + e) = Elem<T>::from_float2(acc[e] * inv, acc[e + 1] * inv);
}

}  // namespace pa
