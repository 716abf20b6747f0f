// paged_decode_q8_pair.cuh -- the one-byte decode (paged_decode_q8.cuh) with
// a CTA per pair of adjacent kv heads.  Included by paged_decode.cu.
//
// With one-byte codes a (token, kv head) row is D bytes: 128 at D = 128.  A
// copy of one block of one kv head is then B rows of 128 bytes at a stride
// of Hkv * D bytes.  Taking two adjacent kv heads per copy makes every token
// row a contiguous 2 * D bytes (256 at D = 128), halves the copies issued,
// and gives each CTA twice the work for the same prologue and epilogue.
//
// Work split: CTA = (kv-head pair, partition, sequence).  Warp w reads head
// 2 * pair + (w & 1) and, with its partner w ^ 1, the partition's blocks
// (w >> 1), (w >> 1) + 2, ...  The two warps of a pair share a ring of
// NSTAGE stages; a stage is one block of both heads, K tile then V tile,
// each [B tokens][2 heads][D] with the 128-byte swizzle at D = 128.  Warp
// (w & 1) == 0 of the pair issues the copies: a stage is refilled once both
// warps have arrived on its "empty" barrier (count 2), and both wait on its
// "full" barrier (the copies' bytes).  Every wait is bounded (pa_common.cuh).
//
// The fused append of a sequence's new token (last partition only) is done
// before any copy: warps 0 and 1 write the row of their kv head, the CTA
// synchronises, and only then are the first copies issued.
#pragma once

#include "paged_decode_q8.cuh"

namespace pa {

// One arrival (no transaction bytes): a consumer handing a stage back.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int D, int BS, int G, bool ROWS>
struct Q8PairShape {
    static constexpr int PAIRS = kWarps / 2;          // warp pairs per CTA
    static constexpr int TILE = 2 * BS * D;           // bytes of one K (or V) tile of both heads
    static constexpr int STAGE = 2 * TILE;
    static constexpr int NSTAGE = STAGE <= 8192 ? 3 : 2;
    static constexpr int RING_BYTES = NSTAGE * STAGE; // one pair's ring
    static constexpr int PT_STRIDE = Q8Shape<D, BS, G, ROWS>::PT_STRIDE;
    static constexpr int PT_BYTES = Q8Shape<D, BS, G, ROWS>::PT_BYTES;
    static constexpr int OFF_PT = PAIRS * RING_BYTES;
    // row scales of a stage: B floats of K for each head, then the same of V
    static constexpr int SC_STAGE = ROWS ? 2 * 2 * BS * 4 : 0;
    static constexpr int OFF_SC = OFF_PT + kWarps * PT_BYTES;
    static constexpr int OFF_BARS = OFF_SC + PAIRS * NSTAGE * SC_STAGE;
    // per pair NSTAGE full + NSTAGE empty barriers, per warp a probe barrier
    static constexpr int BARS = PAIRS * 2 * NSTAGE + kWarps;
    static constexpr int SMEM_BYTES = OFF_BARS + BARS * 8 + 1024;
    static constexpr int EPI_BYTES = kWarps * G * (D + 2) * 4;
    static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
    static_assert(EPI_BYTES <= OFF_BARS, "epilogue fits in the rings");
};

// The partials of the four warps into the CTA's two kv heads' results: head
// h of the pair is the merge of warps h and h + 2 (same as
// merge_warps_and_store, over two warps per head).
template <typename T, int D, int G>
__device__ __forceinline__ void merge_pairs_and_store(
    const float* epi_o, const float* epi_m, const float* epi_l, T* __restrict__ out,
    float* __restrict__ ws_o, float2* __restrict__ ws_ml, int s, int kvh0, int part, int nparts,
    int num_q_heads, int max_parts)
{
    for (int idx = threadIdx.x; idx < 2 * G * D / 8; idx += kThreads) {
        const int hs = idx / (G * D / 8);              // head of the pair
        const int g = (idx / (D / 8)) % G;
        const int d0 = (idx % (D / 8)) * 8;
        const int wa = hs, wb = hs + 2;
        const float ma = epi_m[wa * G + g], mb = epi_m[wb * G + g];
        const float M = fmaxf(ma, mb);
        const float msub = M == -INFINITY ? 0.f : M;
        const float fa = exp2f(ma - msub), fb = exp2f(mb - msub);
        const float L = fmaf(fa, epi_l[wa * G + g], fb * epi_l[wb * G + g]);
        const float4* sa = reinterpret_cast<const float4*>(epi_o + (wa * G + g) * D + d0);
        const float4* sb = reinterpret_cast<const float4*>(epi_o + (wb * G + g) * D + d0);
        const float4 a0 = sa[0], a1 = sa[1], b0 = sb[0], b1 = sb[1];
        float O[8] = {fmaf(fa, a0.x, fb * b0.x), fmaf(fa, a0.y, fb * b0.y),
                      fmaf(fa, a0.z, fb * b0.z), fmaf(fa, a0.w, fb * b0.w),
                      fmaf(fa, a1.x, fb * b1.x), fmaf(fa, a1.y, fb * b1.y),
                      fmaf(fa, a1.z, fb * b1.z), fmaf(fa, a1.w, fb * b1.w)};
        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) O[e] *= inv;
        const int64_t row = static_cast<int64_t>(s) * num_q_heads + (kvh0 + hs) * G + g;
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

// One CTA: (kv-head pair, partition, sequence).
template <typename Codes, typename T, int D, int BS, int G, bool ROWS>
__device__ __forceinline__ void paged_decode_q8_pair_cta(
    const CUtensorMap& tm_k, const CUtensorMap& tm_v, T* __restrict__ out,
    const T* __restrict__ query, const int32_t* __restrict__ block_tables,
    const int32_t* __restrict__ context_lens, int32_t num_q_heads, int32_t max_blocks_per_seq,
    int64_t num_blocks, int32_t max_context_len, float scale_log2, float v_scale,
    int32_t partition_size, int32_t max_parts, float* __restrict__ ws_o,
    float2* __restrict__ ws_ml, int32_t* d_status, int32_t lpt_seqs,
    const T* __restrict__ new_key, const T* __restrict__ new_value, uint8_t* __restrict__ k_cache,
    uint8_t* __restrict__ v_cache, int32_t num_kv_heads, float k_inv, float v_inv, uint32_t probe_us,
    float* __restrict__ k_scales, float* __restrict__ v_scales)
{
    grid_dependency_wait();   // before any global access (see pa_common.cuh)
    using S = Q8PairShape<D, BS, G, ROWS>;
    constexpr int NST = S::NSTAGE;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int kvh0 = 2 * blockIdx.x;
    const int part = blockIdx.y;
    const int s = lpt_seqs > 0
                      ? lpt_sequence(context_lens, block_tables, max_blocks_per_seq, lpt_seqs,
                                     blockIdx.z, reinterpret_cast<int32_t*>(smem))
                      : static_cast<int>(blockIdx.z);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int pair = warp >> 1;
    const int hsel = warp & 1;
    const bool producer = hsel == 0;
    const int kvh = kvh0 + hsel;

    const int blk_begin = blockIdx.y * partition_size / BS;
    // the pair's first chunk of table entries: blocks pair + 2 * lane
    int pre_tbl = -1;
    {
        const int idx = blk_begin + pair + S::PAIRS * lane;
        if (idx < max_blocks_per_seq)
            pre_tbl = block_tables[static_cast<int64_t>(s) * max_blocks_per_seq + idx];
    }
    const int32_t ctx = context_lens[s];
    if (ctx < 0 || ctx > max_context_len ||
        static_cast<int64_t>(ctx) > static_cast<int64_t>(max_blocks_per_seq) * BS) {
        if (part == 0) {
            write_zero_rows<T, D, G>(out, s, kvh0, num_q_heads);
            write_zero_rows<T, D, G>(out, s, kvh0 + 1, num_q_heads);
            if (threadIdx.x == 0) status_or(d_status, PA_STATUS_BAD_CONTEXT);
        }
        return;
    }
    if (ctx == 0) {
        if (part == 0) {
            write_zero_rows<T, D, G>(out, s, kvh0, num_q_heads);
            write_zero_rows<T, D, G>(out, s, kvh0 + 1, num_q_heads);
        }
        return;
    }
    const int tok_begin = part * partition_size;
    if (tok_begin >= ctx) return;
    const int tok_end = min(ctx, tok_begin + partition_size);
    const int nparts = (ctx + partition_size - 1) / partition_size;
    const int nblk = (tok_end - tok_begin + BS - 1) / BS;
    // the pair's blocks: pair, pair + 2, ... of the partition
    const int nk = pair < nblk ? (nblk - pair + S::PAIRS - 1) / S::PAIRS : 0;

    unsigned char* ring = smem + pair * S::RING_BYTES;
    float* rsc = reinterpret_cast<float*>(smem + S::OFF_SC) + pair * NST * (S::SC_STAGE / 4);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BARS);
    uint64_t* full = bars + pair * 2 * NST;
    uint64_t* empty = full + NST;
    uint64_t* probe = bars + S::PAIRS * 2 * NST + warp;
    if (lane == 0) {
        if (producer) {
#pragma unroll
            for (int st = 0; st < NST; ++st) {
                mbar_init(&full[st], 1);
                mbar_init(&empty[st], 2);
            }
        }
        mbar_init(probe, 1);
        fence_barrier_init();
    }
    // the fused append of the sequence's new token: warps 0 and 1 write the
    // row of their kv head before any copy of the CTA is issued
    const bool appends = new_key != nullptr && part == nparts - 1;
    if (appends && warp < 2) {
        const int32_t phys = block_tables[static_cast<int64_t>(s) * max_blocks_per_seq + (ctx - 1) / BS];
        if (phys >= 0 && static_cast<int64_t>(phys) < num_blocks) {
            if constexpr (ROWS)
                append_row_warp_rowscale<Codes, T, D, BS>(new_key, new_value, k_cache, v_cache,
                                                          k_scales, v_scales, s, kvh, num_kv_heads,
                                                          ctx - 1, phys, lane);
            else
                append_row_warp_q8<Codes, T, D, BS>(new_key, new_value, k_cache, v_cache, s, kvh,
                                                    num_kv_heads, ctx - 1, phys, k_inv, v_inv, lane);
        } else if (lane == 0) {
            status_or(d_status, PA_STATUS_BAD_SLOT);
        }
    }
    __syncthreads();   // barriers initialised, appended rows written
    if (appends) fence_proxy_async_global();

    const int32_t* table = block_tables + static_cast<int64_t>(s) * max_blocks_per_seq + blk_begin;
    // a table chunk: lane l holds the physical block of the pair's block
    // 32 * chunk + l, or -1 past the pair's blocks and for an id outside the pool
    auto valid = [&](int32_t phys) -> int {
        return phys >= 0 && static_cast<int64_t>(phys) < num_blocks ? phys : -1;
    };
    auto load_table = [&](int chunk) -> int {
        const int kk = chunk * 32 + lane;
        return kk < nk ? valid(table[pair + S::PAIRS * kk]) : -1;
    };
    int prod_chunk = 0, cons_chunk = 0;
    int prod_tbl = lane < nk ? valid(pre_tbl) : -1;
    int cons_tbl = prod_tbl;
    // producer: copies of the pair's block k into stage st (both heads)
    auto issue = [&](int k, int st) {
        const int chunk = k >> 5;
        if (chunk != prod_chunk) {
            prod_tbl = load_table(chunk);
            prod_chunk = chunk;
        }
        const int phys = __shfl_sync(kFullMask, prod_tbl, k & 31);
        if (lane == 0) {
            fence_proxy_async_smem();
            if (phys >= 0) {
                mbar_arrive_expect_tx(&full[st], 2u * S::TILE + static_cast<uint32_t>(S::SC_STAGE));
                unsigned char* dst = ring + st * S::STAGE;
                tma_load_4d(dst, &tm_k, 0, kvh0, 0, phys, &full[st]);
                tma_load_4d(dst + S::TILE, &tm_v, 0, kvh0, 0, phys, &full[st]);
                if constexpr (ROWS) {
                    // the block's B row scales of both heads: one contiguous run each
                    const int64_t so = (static_cast<int64_t>(phys) * num_kv_heads + kvh0) * BS;
                    float* sc = rsc + st * (S::SC_STAGE / 4);
                    bulk_copy_g2s(sc, k_scales + so, 2 * BS * 4, &full[st]);
                    bulk_copy_g2s(sc + 2 * BS, v_scales + so, 2 * BS * 4, &full[st]);
                }
            } else {
                status_or(d_status, PA_STATUS_BAD_BLOCK);
                mbar_arrive_expect_tx(&full[st], 0u);
            }
        }
    };
    const int prologue = min(nk, NST);
    if (producer)
        for (int k = 0; k < prologue; ++k) issue(k, k);
    int issued = prologue;

    Q8Warp<Codes, T, D, BS, G, ROWS, 2> w;
    w.grp = lane >> 2;
    w.tig = lane & 3;
    w.hsel = hsel;
    w.pt_addr = smem_u32(smem + S::OFF_PT + warp * S::PT_BYTES) + (lane & 7) * S::PT_STRIDE +
                ((lane >> 3) & 1) * 16;
    w.reset();
    w.load_q(query, s, kvh, num_q_heads);

    bool aborted = nk > 0 && probe_gives_up(probe, probe_us);
    int first_pending = 0;
    int st = 0;
    uint32_t phase = 0;
    int t0 = tok_begin + pair * BS;             // first token of the pair's block k
    for (int k = 0; k < (aborted ? 0 : nk); ++k) {
        if (!mbar_wait_warp(&full[st], phase)) {
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
        const int nv = phys >= 0 ? min(BS, tok_end - t0) : 0;
        const unsigned char* kt = ring + st * S::STAGE;
        const float* sc = rsc + st * (S::SC_STAGE / 4);
        w.block(kt, kt + S::TILE, nv, scale_log2, sc + hsel * BS, sc + 2 * BS + hsel * BS);
        if (k % kBiasFlushBlocks == kBiasFlushBlocks - 1) w.flush_bias();
        __syncwarp();   // every lane is done with this stage
        if (lane == 0) mbar_arrive(&empty[st]);
        if (producer && issued < nk) {
            // refill the stage once the partner warp is done with it too
            if (!mbar_wait_warp(&empty[st], phase)) {
                aborted = true;
                first_pending = k + 1;
                break;
            }
            issue(issued, st);
            ++issued;
        }
        t0 += S::PAIRS * BS;
        if (++st == NST) {
            st = 0;
            phase ^= 1u;
        }
    }

    // only the producer has copies of its own to wait for
    if (aborted && producer) drain_after_timeout<NST>(full, first_pending, issued, d_status);
    else if (aborted && threadIdx.x % 32 == 0) status_or(d_status, PA_STATUS_TIMEOUT);

    // every warp is done with the rings, unless one gave up waiting
    if (__syncthreads_or(aborted)) {
        store_aborted_rows<T, D, G>(out, ws_o, ws_ml, s, kvh0, part, nparts, num_q_heads, max_parts);
        store_aborted_rows<T, D, G>(out, ws_o, ws_ml, s, kvh0 + 1, part, nparts, num_q_heads,
                                    max_parts);
        return;
    }
    float* epi_o = reinterpret_cast<float*>(smem);   // [warp][g][D]
    float* epi_m = epi_o + kWarps * G * D;
    float* epi_l = epi_m + kWarps * G;
    w.store(epi_o, epi_m, epi_l, warp, ROWS ? w.vref : v_scale);
    __syncthreads();
    merge_pairs_and_store<T, D, G>(epi_o, epi_m, epi_l, out, ws_o, ws_ml, s, kvh0, part, nparts,
                                   num_q_heads, max_parts);
}

template <typename T, int D, int BS, int G, bool ROWS>
__global__ void __launch_bounds__(kThreads, 4) paged_decode_fp8_pair_kernel(PA_Q8_KERNEL_PARAMS)
{
    paged_decode_q8_pair_cta<E4m3Codes, T, D, BS, G, ROWS>(PA_Q8_KERNEL_ARGS);
}

template <typename T, int D, int BS, int G, bool ROWS>
__global__ void __launch_bounds__(kThreads, 4) paged_decode_int8_pair_kernel(PA_Q8_KERNEL_PARAMS)
{
    paged_decode_q8_pair_cta<Int8Codes, T, D, BS, G, ROWS>(PA_Q8_KERNEL_ARGS);
}

#undef PA_Q8_KERNEL_PARAMS
#undef PA_Q8_KERNEL_ARGS

}  // namespace pa
