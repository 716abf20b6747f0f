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
// One launch covers two kinds of work item (blockIdx.z):
//   z <  num_groups : the shared prefix [0, L) of group z, every member's
//                     query rows at once (rows = members x G <= 8), K/V
//                     through the first member's block table;
//   z >= num_groups : the private suffix [L, ctx) of one sequence.
// Both are split into context partitions and leave (max, exp-sum,
// normalised output) partials in the workspace; a reduction kernel merges
// each row's prefix and suffix partials with the rule of §5.1.

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
    static constexpr int SMEM_BYTES = OFF_BARS + kWarps * NSTAGE * 8 + 1024;
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

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads, 3) paged_decode_shared_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const T* __restrict__ query, const int32_t* __restrict__ block_tables,
    const int32_t* __restrict__ context_lens, const int32_t* __restrict__ prefix_lens,
    int32_t num_groups, int32_t group_size, int32_t G, int32_t num_q_heads,
    int32_t max_blocks_per_seq, int64_t num_blocks, int32_t max_context_len,
    int32_t max_prefix_len, float scale_log2, int32_t partition_size, int32_t prefix_slots,
    int32_t slots, float* __restrict__ ws_o, float2* __restrict__ ws_ml, int32_t* d_status)
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

    // ---- the work item: rows, token range, block table, output slot ----
    const bool is_prefix = z < num_groups;
    const int group = is_prefix ? z : (z - num_groups) / group_size;
    const int seq0 = is_prefix ? z * group_size : z - num_groups;   // first row's sequence
    const int rows = is_prefix ? group_size * G : G;
    const int32_t L = prefix_lens[group];
    if (!prefix_ok(context_lens, L, group, group_size, BS, max_prefix_len, max_context_len,
                   max_tokens))
        return;                              // the reduction reports it and writes zero rows
    const int32_t ctx_end = is_prefix ? L : context_lens[seq0];
    const int32_t start = is_prefix ? 0 : L;
    const int tok_begin = start + part * partition_size;
    if (tok_begin >= ctx_end) return;
    const int tok_end = min(ctx_end, tok_begin + partition_size);
    const int slot = is_prefix ? part : prefix_slots + part;
    const int blk_begin = tok_begin / BS;
    const int nblk = (tok_end - tok_begin + BS - 1) / BS;
    const int nk = warp < nblk ? (nblk - warp + kWarps - 1) / kWarps : 0;

    unsigned char* wstage = smem + warp * S::WARP_STAGE_BYTES;
    uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + S::OFF_BARS) + warp * S::NSTAGE;
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < S::NSTAGE; ++st) mbar_init(&wbar[st], 1);
        fence_barrier_init();
    }
    __syncwarp();

    const int32_t* table = block_tables + static_cast<int64_t>(seq0) * max_blocks_per_seq + blk_begin;
    const int members = is_prefix ? group_size : 1;
    // One table entry per lane, 32 blocks per load; for a prefix, every
    // member's entry must name the same physical block.
    auto load_table = [&](int chunk) -> int {
        const int kk = chunk * 32 + lane;
        if (kk >= nk) return -1;
        const int j = warp + kWarps * kk;
        const int32_t e = table[j];
        bool same = true;
        for (int m = 1; m < members; ++m)
            same &= table[static_cast<int64_t>(m) * max_blocks_per_seq + j] == e;
        if (!same) status_or(d_status, PA_STATUS_BAD_BLOCK);
        return e;
    };
    int prod_chunk = 0, cons_chunk = 0;
    int prod_tbl = load_table(0);
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
            const int tv = nv - t0;
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

    if (aborted) {
        if (lane == 0) status_or(d_status, PA_STATUS_TIMEOUT);
        for (int k = first_pending; k < issued; ++k) {
            const int st = k % S::NSTAGE;
            mbar_wait_bounded(&wbar[st], (k / S::NSTAGE) & 1);
        }
    }

    l_run += __shfl_xor_sync(kFullMask, l_run, 1);
    l_run += __shfl_xor_sync(kFullMask, l_run, 2);

    __syncthreads();
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

    // merge the warps in a fixed order; every row leaves a partial
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
        const int64_t row = static_cast<int64_t>(seq0 + r / G) * num_q_heads + kvh * G + r % G;
        const int64_t prow = row * slots + slot;
        float4* dst = reinterpret_cast<float4*>(ws_o + prow * D + d0);
        dst[0] = make_float4(O[0] * inv, O[1] * inv, O[2] * inv, O[3] * inv);
        dst[1] = make_float4(O[4] * inv, O[5] * inv, O[6] * inv, O[7] * inv);
        if (d0 == 0) ws_ml[prow] = make_float2(M, Lsum);
    }
}

// One warp per (sequence, query head): merge the prefix partials (slots
// [0, ceil(L / P))) and the suffix partials (slots [prefix_slots,
// prefix_slots + ceil((ctx - L) / P))) into the output row.
template <typename T, int D>
__global__ void __launch_bounds__(kReduceRowsPerCta * 32) paged_decode_shared_reduce_kernel(
    T* __restrict__ out, const float* __restrict__ ws_o, const float2* __restrict__ ws_ml,
    const int32_t* __restrict__ context_lens, const int32_t* __restrict__ prefix_lens,
    int32_t num_seqs, int32_t group_size, int32_t num_q_heads, int32_t max_context_len,
    int32_t max_blocks_per_seq, int32_t block_size, int32_t max_prefix_len,
    int32_t partition_size, int32_t prefix_slots, int32_t slots, int32_t* d_status)
{
    grid_dependency_wait();
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kReduceRowsPerCta + (threadIdx.x >> 5);
    if (row >= static_cast<int64_t>(num_seqs) * num_q_heads) return;
    const int s = static_cast<int>(row / num_q_heads);
    const int z = s / group_size;
    const int32_t ctx = context_lens[s];
    const int32_t L = prefix_lens[z];
    T* dst = out + row * D + lane * EPL;
    if (!prefix_ok(context_lens, L, z, group_size, block_size, max_prefix_len, max_context_len,
                   max_blocks_per_seq * block_size)) {
        if (lane == 0) status_or(d_status, PA_STATUS_BAD_CONTEXT);
#pragma unroll
        for (int e = 0; e < EPL; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = 0u;
        return;
    }
    const int n_pre = (L + partition_size - 1) / partition_size;
    const int n_suf = (ctx - L + partition_size - 1) / partition_size;
    const int n = n_pre + n_suf;
    auto slot_of = [&](int i) { return i < n_pre ? i : prefix_slots + (i - n_pre); };
    const float2* ml = ws_ml + row * slots;
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) M = fmaxf(M, ml[slot_of(i)].x);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, m));
    const float msub = M == -INFINITY ? 0.f : M;
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    float W = 0.f;
    const float* orow = ws_o + row * slots * D + lane * EPL;
    for (int i = 0; i < n; ++i) {
        const int sl = slot_of(i);
        const float2 v = ml[sl];
        const float w = v.y * exp2f(v.x - msub);
        W += w;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, orow[static_cast<int64_t>(sl) * D + e], acc[e]);
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
    for (int e = 0; e < EPL; e += 2)
        *reinterpret_cast<uint32_t*>(dst + e) = Elem<T>::from_float2(acc[e] * inv, acc[e + 1] * inv);
}

}  // namespace pa
