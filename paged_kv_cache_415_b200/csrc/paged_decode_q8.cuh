// paged_decode_q8.cuh -- decode over K/V pools of one-byte codes (e4m3 or
// int8, pa_codes.cuh) with per-pool scales.  Included by paged_decode.cu.
//
// "PagedAttention：大模型KV Cache分页管理优化实践" §7 and "vLLM用虚拟内存分页思想
// 管理KV Cache" (工程实践与局限) name low-precision storage of the cached blocks;
// at one byte per element every decode step moves half the bytes.
//
// Same work split, TMA pipeline, online softmax and merge as the 16-bit
// kernels; the tiles arrive as bytes (B rows x D codes, 128-byte swizzle for
// D = 128) and never go back to shared memory in a wider type.  Both
// contractions run on the tensor cores (mma.sync m16n8k16, fp16 in, fp32
// accumulate) with the cache tile as the A operand and the heads of the
// group as the 8 columns of N, so a lone query head wastes 7/8 of an MMA
// rather than 15/16:
//
//   S^T [16 tokens x 8 heads]  = K [16 x D] . Q^T [D x 8]
//   O^T [D x 8 heads]         += V^T [D x 16 tokens] . P^T [16 x 8]
//
// Each lane reads its A fragments straight from the byte tile, pairs codes
// with byte permutes where two tokens share a register (V^T), and widens
// them exactly to fp16 (Codes::widen4: one cvt per pair for e4m3; for int8
// a byte permute per pair that yields 1152 + c).  The int8 bias is removed
// once per head, not per code: every score of head h carries 1152 * sum_d
// q[h][d] (subtracted from the scores; the sum is taken once per CTA from
// the fp16 query the MMA reads), and the output carries 1152 * sum_t p_t
// (subtracted every kBiasFlushBlocks blocks and in the epilogue, from the
// sum of the P values the MMA read, so the accumulator never holds more
// than a few blocks' worth of it).  The contraction index
// may be permuted freely as long as both operands follow it, so every lane
// reads whole 16-byte runs of one token row.  P moves from the accumulator
// layout (tokens x heads) to the B layout (heads x tokens) through a
// 384-byte shared tile with stmatrix.trans / ldmatrix.  Scales: k_scale
// folds into the score scale, v_scale into the output.  The query is
// rounded once to fp16 (exact for fp16 queries).
//
// Row-scaled pools (ROWS = true): every (token, kv head) row has its own
// fp32 scale, in pools [num_blocks][num_kv_heads][block_size] beside the
// codes.  A block's B scales of K and of V for this kv head are one
// contiguous run each; two more bulk copies bring them into the stage with
// the tiles, counted on the same mbarrier.  The score of token t is
// multiplied by its K row scale after the MMA.  The V row scale folds into
// P: the B operand of O^T += V^T . P^T is p_t * (vs_t / R) in fp16, where R
// is the largest V row scale seen so far by the warp -- a running reference
// rescaled like the running max of the softmax -- so P stays in fp16's
// normal range whatever the scales' magnitude; the epilogue multiplies the
// output by R.
#pragma once

#include "decode_common.cuh"
#include "pa_codes.cuh"

namespace pa {

template <int D, int BS, int G, bool ROWS = false>
struct Q8Shape {
    static constexpr int SLICES = BS / 16;           // 16-token MMA slices per block
    static constexpr int KW = D / 16;                // k-steps of S^T; 4-code words per K row per lane
    static constexpr int KV16 = KW / 4;              // 16-byte K loads per row per lane
    static constexpr int DPT = D / 8;                // output dims per lane (V^T rows)
    static constexpr int VQ = DPT / 4;               // 4-code words per V row per lane
    static constexpr int MT = D / 16;                // m-tiles of V^T
    static constexpr bool SWIZZLE = (D == 128);      // 128-byte rows, 128B TMA swizzle
    static constexpr int TILE = BS * D;              // bytes of one K (or V) tile of one head
    static constexpr int STAGE = 2 * TILE;
    static constexpr int NSTAGE = STAGE <= 4096 ? 3 : 2;
    static constexpr int PT_STRIDE = 48;             // bytes per head row of the P^T tile
    static constexpr int PT_BYTES = 8 * PT_STRIDE;
    static constexpr int WARP_BYTES = NSTAGE * STAGE;
    static constexpr int OFF_PT = kWarps * WARP_BYTES;
    // row scales of a stage: B floats of K, then B of V
    static constexpr int SC_STAGE = ROWS ? 2 * BS * 4 : 0;
    static constexpr int OFF_SC = OFF_PT + kWarps * PT_BYTES;
    static constexpr int OFF_BARS = OFF_SC + kWarps * NSTAGE * SC_STAGE;
    // + a probe barrier per warp, + alignment slack
    static constexpr int SMEM_BYTES = OFF_BARS + kWarps * (NSTAGE + 1) * 8 + 1024;
    static constexpr int EPI_BYTES = kWarps * G * (D + 2) * 4;
    static_assert(BS % 16 == 0 && (D == 64 || D == 128), "whole 16-token slices");
    static_assert(G >= 1 && G <= 8, "heads are the 8 columns of N");
    static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
    static_assert(EPI_BYTES <= OFF_BARS, "epilogue fits in the warp buffers");
};

// Byte offset of (row, byte) in a tile; byte is a multiple of 8 within the
// row.  D = 128: 128-byte rows with the TMA 128B swizzle (16-byte chunk c
// of row r sits at chunk c ^ (r & 7)); D = 64: dense 64-byte rows.
template <int D>
__device__ __forceinline__ uint32_t q8_tile_off(int row, int byte)
{
    if constexpr (D == 128)
        return static_cast<uint32_t>(row * 128 + ((((byte >> 4) ^ (row & 7)) << 4) | (byte & 15)));
    else
        return static_cast<uint32_t>(row * D + byte);
}

// Blocks between two removals of the int8 bias from the output accumulator
// (Q8Warp::flush_bias).
constexpr int kBiasFlushBlocks = 8;

// 2^x with the special-function unit's approximation (flushes subnormal
// results to zero); the probabilities it produces are rounded to fp16 next.
__device__ __forceinline__ float q8_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void stmatrix_x2_trans(uint32_t smem_addr, uint32_t r0, uint32_t r1)
{
    asm volatile("stmatrix.sync.aligned.m8n8.x2.trans.shared.b16 [%0], {%1, %2};"
                 :
                 : "r"(smem_addr), "r"(r0), "r"(r1)
                 : "memory");
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t& r0, uint32_t& r1, uint32_t smem_addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(smem_addr)
                 : "memory");
}

// Fused cache write for quantised pools: the warp that loads the block
// holding a sequence's new token first encodes that token's K and V row for
// its kv head exactly as the cache-write kernel does (fp32(x) * fp32(1 /
// scale), then Codes::encode2) and stores the codes, then makes the writes
// visible to the tensor-copy engine before the block's tiles are requested.
// Warp-uniform.
template <typename Codes, typename T, int D, int BS>
__device__ __forceinline__ void append_row_warp_q8(
    const T* __restrict__ new_key, const T* __restrict__ new_value, uint8_t* __restrict__ k_cache,
    uint8_t* __restrict__ v_cache, int s, int kvh, int num_kv_heads, int32_t pos, int32_t phys,
    float k_inv, float v_inv, int lane)
{
    const int64_t slot = static_cast<int64_t>(phys) * BS + pos % BS;
    const int64_t src = (static_cast<int64_t>(s) * num_kv_heads + kvh) * D;
    const int64_t dst = (slot * num_kv_heads + kvh) * D;
    if (lane < D / 8) {
        const uint4 kv = ld_nc_v4(new_key + src + lane * 8);
        const uint4 vv = ld_nc_v4(new_value + src + lane * 8);
        *reinterpret_cast<uint2*>(k_cache + dst + lane * 8) = encode8<Codes, T>(kv, k_inv);
        *reinterpret_cast<uint2*>(v_cache + dst + lane * 8) = encode8<Codes, T>(vv, v_inv);
        fence_proxy_async_global();
    }
    __syncwarp();
    fence_proxy_async_global();
}

// The same for row-scaled pools: the warp quantises the row with a scale of
// its own (quantise_row_warp, as the row-scaled cache-write kernel does) and
// stores the codes and the scale, then fences both for the copy engine.
template <typename Codes, typename T, int D, int BS>
__device__ __forceinline__ void append_row_warp_rowscale(
    const T* __restrict__ new_key, const T* __restrict__ new_value, uint8_t* __restrict__ k_cache,
    uint8_t* __restrict__ v_cache, float* __restrict__ k_scales, float* __restrict__ v_scales,
    int s, int kvh, int num_kv_heads, int32_t pos, int32_t phys, int lane)
{
    const int64_t slot = static_cast<int64_t>(phys) * BS + pos % BS;
    const int64_t src = (static_cast<int64_t>(s) * num_kv_heads + kvh) * D;
    const int64_t dst = (slot * num_kv_heads + kvh) * D;
    uint4 kx = make_uint4(0, 0, 0, 0), vx = make_uint4(0, 0, 0, 0);
    if (lane < D / 8) {
        kx = ld_nc_v4(new_key + src + lane * 8);
        vx = ld_nc_v4(new_value + src + lane * 8);
    }
    float ks, vs;
    const uint2 kc = quantise_row_warp<Codes, T, D>(kx, ks);
    const uint2 vc = quantise_row_warp<Codes, T, D>(vx, vs);
    if (lane < D / 8) {
        *reinterpret_cast<uint2*>(k_cache + dst + lane * 8) = kc;
        *reinterpret_cast<uint2*>(v_cache + dst + lane * 8) = vc;
    }
    if (lane == 0) {
        const int64_t si = (static_cast<int64_t>(phys) * num_kv_heads + kvh) * BS + pos % BS;
        k_scales[si] = ks;
        v_scales[si] = vs;
    }
    fence_proxy_async_global();
    __syncwarp();
    fence_proxy_async_global();
}

template <int D>
__device__ __forceinline__ void load_words(const unsigned char* tile, int row, int byte,
                                           uint32_t (&w)[4])
{
    const uint4 v = *reinterpret_cast<const uint4*>(tile + q8_tile_off<D>(row, byte));
    w[0] = v.x;
    w[1] = v.y;
    w[2] = v.z;
    w[3] = v.w;
}

// One warp's share of a (sequence, kv head, partition) unit: Q^T fragments,
// the O^T accumulators and the online-softmax state of heads 2*tig and
// 2*tig + 1 (rows of N), and the code that consumes one block of K/V bytes.
//
// HP is the number of kv heads a tile holds: 1, or 2 when one copy brings
// two adjacent kv heads (their rows interleave: line 2r + h of the tile is
// token r of head h), hsel the head this warp reads.
template <typename Codes, typename T, int D, int BS, int G, bool ROWS = false, int HP = 1>
struct Q8Warp {
    using S = Q8Shape<D, BS, G, ROWS>;
    int grp, tig;
    int hsel = 0;                   // HP = 2: which of the tile's two heads
    uint32_t pt_addr;               // this lane's row of the P^T staging tile
    uint32_t qb[S::KW][2];
    float o[S::MT][4];
    float m_run0, m_run1;           // running maxima (log2 units)
    float l_run0, l_run1;           // this lane's share of the exp-sums
    float vref, vinv;               // ROWS: running reference of the V row scales, 1 / it
    float e0, e1;                   // kBias * sum_d q[h][d] of heads 2tig, 2tig + 1
    float ps_run0, ps_run1;         // int8: sum of the P values fed to the MMA since the last flush

    // tile line of token row r
    __device__ __forceinline__ int line(int r) const { return HP == 1 ? r : r * HP + hsel; }

    __device__ __forceinline__ void reset()
    {
#pragma unroll
        for (int mt = 0; mt < S::MT; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;
        m_run0 = m_run1 = -INFINITY;
        l_run0 = l_run1 = 0.f;
        vref = vinv = 0.f;
        e0 = e1 = 0.f;
        ps_run0 = ps_run1 = 0.f;
    }

    // Q^T as B fragments, fp16: k-step j holds head grp's dims
    // (D/4)*tig + 4j .. +3, the same dims the lane's K words carry.
    __device__ __forceinline__ void load_q(const T* __restrict__ query, int s, int kvh,
                                           int num_q_heads)
    {
        const T* qrow = query + (static_cast<int64_t>(s) * num_q_heads + kvh * G + grp) * D +
                        (D / 4) * tig;
#pragma unroll
        for (int j = 0; j < S::KW; ++j) {
            uint32_t b0 = 0u, b1 = 0u;
            if (grp < G) {
                const uint2 w = *reinterpret_cast<const uint2*>(qrow + 4 * j);
                const float2 f0 = Elem<T>::to_float2(w.x);
                const float2 f1 = Elem<T>::to_float2(w.y);
                b0 = Elem<__half>::from_float2(f0.x, f0.y);
                b1 = Elem<__half>::from_float2(f1.x, f1.y);
            }
            qb[j][0] = b0;
            qb[j][1] = b1;
        }
        if constexpr (Codes::kBias != 0.f) {
            // sum of head grp's fp16 query (the values the MMA reads), then
            // the bias every score of heads 2tig and 2tig + 1 carries
            float qs = 0.f;
#pragma unroll
            for (int j = 0; j < S::KW; ++j) {
                const float2 a = Elem<__half>::to_float2(qb[j][0]);
                const float2 b = Elem<__half>::to_float2(qb[j][1]);
                qs += (a.x + a.y) + (b.x + b.y);
            }
            qs += __shfl_xor_sync(kFullMask, qs, 1);
            qs += __shfl_xor_sync(kFullMask, qs, 2);
            e0 = Codes::kBias * __shfl_sync(kFullMask, qs, 8 * tig);
            e1 = Codes::kBias * __shfl_sync(kFullMask, qs, 8 * tig + 4);
        }
    }

    // One block: kt / vt are its K and V byte tiles, nv its valid tokens;
    // with ROWS, ksc / vsc its B row scales of K and of V.
    __device__ __forceinline__ void block(const unsigned char* kt, const unsigned char* vt, int nv,
                                          float scale_log2, const float* ksc = nullptr,
                                          const float* vsc = nullptr)
    {
#pragma unroll 1
        for (int sl = 0; sl < S::SLICES; ++sl) {
            const int t0 = sl * 16;
            const int tv = nv - t0;             // valid tokens of this slice
            if (tv <= 0) break;

            // ---- S^T = K . Q^T: rows grp and grp + 8 of the slice ----
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int h = 0; h < S::KV16; ++h) {
                uint32_t w0[4], w1[4];
                load_words<D>(kt, line(t0 + grp), (D / 4) * tig + 16 * h, w0);
                load_words<D>(kt, line(t0 + grp + 8), (D / 4) * tig + 16 * h, w1);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = 4 * h + i;
                    uint32_t a0, a2, a1, a3;
                    Codes::widen4(w0[i], a0, a2);
                    Codes::widen4(w1[i], a1, a3);
                    if (j & 1)
                        mma_16816<__half>(sb, a0, a1, a2, a3, qb[j][0], qb[j][1]);
                    else
                        mma_16816<__half>(sa, a0, a1, a2, a3, qb[j][0], qb[j][1]);
                }
            }
            // this lane: tokens grp (x0, x1) and grp + 8 (x2, x3); heads 2tig, 2tig + 1
            float sla = scale_log2, slb = scale_log2;
            if constexpr (ROWS) {               // each token's K row scale
                sla *= ksc[t0 + grp];
                slb *= ksc[t0 + grp + 8];
            }
            const float x0 = grp < tv ? ((sa[0] + sb[0]) - e0) * sla : -INFINITY;
            const float x1 = grp < tv ? ((sa[1] + sb[1]) - e1) * sla : -INFINITY;
            const float x2 = grp + 8 < tv ? ((sa[2] + sb[2]) - e0) * slb : -INFINITY;
            const float x3 = grp + 8 < tv ? ((sa[3] + sb[3]) - e1) * slb : -INFINITY;

            // ---- online softmax per head over the slice's 16 tokens ----
            float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
            for (int m = 4; m < 32; m <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, m));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, m));
            }
            const float mn0 = fmaxf(m_run0, mx0), mn1 = fmaxf(m_run1, mx1);
            const float ms0 = mn0 == -INFINITY ? 0.f : mn0;
            const float ms1 = mn1 == -INFINITY ? 0.f : mn1;
            const float c0 = q8_exp2(m_run0 - ms0), c1 = q8_exp2(m_run1 - ms1);
            m_run0 = mn0;
            m_run1 = mn1;
            uint32_t pk0, pk1;
            float2 cc = make_float2(c0, c1);
            if constexpr (ROWS) {
                // V row scales of the slice's tokens relative to the running
                // reference (rows past the context weigh 0); the reference
                // grows to the slice's largest scale and rescales O like a
                // change of the running max does
                const float va = grp < tv ? vsc[t0 + grp] : 0.f;
                const float vb = grp + 8 < tv ? vsc[t0 + grp + 8] : 0.f;
                float vmax = fmaxf(va, vb);
#pragma unroll
                for (int m = 4; m < 32; m <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(kFullMask, vmax, m));
                if (vmax > vref) {              // warp-uniform
                    const float fr = vref / vmax;
                    cc.x *= fr;
                    cc.y *= fr;
                    vref = vmax;
                    vinv = 1.f / vmax;
                }
                const float p0 = q8_exp2(x0 - ms0), p1 = q8_exp2(x1 - ms1);
                const float p2 = q8_exp2(x2 - ms0), p3 = q8_exp2(x3 - ms1);
                l_run0 = l_run0 * c0 + (p0 + p2);
                l_run1 = l_run1 * c1 + (p1 + p3);
                const float ra = va * vinv, rb = vb * vinv;
                pk0 = Elem<__half>::from_float2(p0 * ra, p1 * ra);
                pk1 = Elem<__half>::from_float2(p2 * rb, p3 * rb);
                if constexpr (Codes::kBias != 0.f) {   // the P values the MMA reads
                    const float2 f0 = Elem<__half>::to_float2(pk0), f1 = Elem<__half>::to_float2(pk1);
                    ps_run0 = ps_run0 * cc.x + (f0.x + f1.x);
                    ps_run1 = ps_run1 * cc.y + (f0.y + f1.y);
                }
            } else {
                // P rounds to fp16 for the tensor cores; the sums use the rounded values
                pk0 = Elem<__half>::from_float2(q8_exp2(x0 - ms0), q8_exp2(x1 - ms1));
                pk1 = Elem<__half>::from_float2(q8_exp2(x2 - ms0), q8_exp2(x3 - ms1));
                const float2 r0 = Elem<__half>::to_float2(pk0), r1 = Elem<__half>::to_float2(pk1);
                l_run0 = l_run0 * c0 + (r0.x + r1.x);
                l_run1 = l_run1 * c1 + (r0.y + r1.y);
                if constexpr (Codes::kBias != 0.f) {   // the P values the MMA reads
                    ps_run0 = ps_run0 * c0 + (r0.x + r1.x);
                    ps_run1 = ps_run1 * c1 + (r0.y + r1.y);
                }
            }
            // once the running maxima settle, most slices leave them unchanged
            if (__any_sync(kFullMask, cc.x != 1.f || cc.y != 1.f)) {
#pragma unroll
                for (int mt = 0; mt < S::MT; ++mt) {
                    float2 u = __fmul2_rn(make_float2(o[mt][0], o[mt][1]), cc);
                    float2 v = __fmul2_rn(make_float2(o[mt][2], o[mt][3]), cc);
                    o[mt][0] = u.x;
                    o[mt][1] = u.y;
                    o[mt][2] = v.x;
                    o[mt][3] = v.y;
                }
            }

            // ---- P (tokens x heads) -> P^T B fragments (heads x tokens) ----
            uint32_t pb0, pb1;
            __syncwarp();
            stmatrix_x2_trans(pt_addr, pk0, pk1);
            __syncwarp();
            ldmatrix_x2(pb0, pb1, pt_addr);

            // ---- O^T += V^T . P^T: tokens 2tig, 2tig+1, 2tig+8, 2tig+9 ----
            const int ta = t0 + 2 * tig;
            uint32_t va[S::VQ], vb[S::VQ], vc[S::VQ], vd[S::VQ];
            if constexpr (S::VQ == 4) {
                uint32_t w[4];
                load_words<D>(vt, line(ta), S::DPT * grp, w);
#pragma unroll
                for (int q = 0; q < 4; ++q) va[q] = w[q];
                load_words<D>(vt, line(ta + 1), S::DPT * grp, w);
#pragma unroll
                for (int q = 0; q < 4; ++q) vb[q] = w[q];
                load_words<D>(vt, line(ta + 8), S::DPT * grp, w);
#pragma unroll
                for (int q = 0; q < 4; ++q) vc[q] = w[q];
                load_words<D>(vt, line(ta + 9), S::DPT * grp, w);
#pragma unroll
                for (int q = 0; q < 4; ++q) vd[q] = w[q];
            } else {
                const uint2 a = *reinterpret_cast<const uint2*>(vt + q8_tile_off<D>(line(ta), S::DPT * grp));
                const uint2 b = *reinterpret_cast<const uint2*>(vt + q8_tile_off<D>(line(ta + 1), S::DPT * grp));
                const uint2 c = *reinterpret_cast<const uint2*>(vt + q8_tile_off<D>(line(ta + 8), S::DPT * grp));
                const uint2 d = *reinterpret_cast<const uint2*>(vt + q8_tile_off<D>(line(ta + 9), S::DPT * grp));
                va[0] = a.x; va[1] = a.y;
                vb[0] = b.x; vb[1] = b.y;
                vc[0] = c.x; vc[1] = c.y;
                vd[0] = d.x; vd[1] = d.y;
            }
            if (tv < 16) {   // rows past the context may hold any code (NaN included)
                const int ra = 2 * tig;
#pragma unroll
                for (int q = 0; q < S::VQ; ++q) {
                    va[q] = ra < tv ? va[q] : 0u;
                    vb[q] = ra + 1 < tv ? vb[q] : 0u;
                    vc[q] = ra + 8 < tv ? vc[q] : 0u;
                    vd[q] = ra + 9 < tv ? vd[q] : 0u;
                }
            }
#pragma unroll
            for (int q = 0; q < S::VQ; ++q) {
                // token pairs per dim: [b1 a1 b0 a0] and [b3 a3 b2 a2]
                const uint32_t lo_ab = __byte_perm(va[q], vb[q], 0x5140);
                const uint32_t hi_ab = __byte_perm(va[q], vb[q], 0x7362);
                const uint32_t lo_cd = __byte_perm(vc[q], vd[q], 0x5140);
                const uint32_t hi_cd = __byte_perm(vc[q], vd[q], 0x7362);
                uint32_t a0, a1, a2, a3;
                // m-tile 2q: rows grp / grp + 8 are dims DPT*grp + 4q + 0 / + 1
                Codes::widen4(lo_ab, a0, a1);
                Codes::widen4(lo_cd, a2, a3);
                mma_16816<__half>(o[2 * q], a0, a1, a2, a3, pb0, pb1);
                // m-tile 2q + 1: dims + 2 / + 3
                Codes::widen4(hi_ab, a0, a1);
                Codes::widen4(hi_cd, a2, a3);
                mma_16816<__half>(o[2 * q + 1], a0, a1, a2, a3, pb0, pb1);
            }
        }
    }

    // int8 codes: every V value the MMA read carried the bias, so O holds
    // kBias times the sum of the P values it was weighted with.  Remove what
    // has gathered since the last call (the sum over the warp's lanes) and
    // start that sum again.  Called every kBiasFlushBlocks blocks and before
    // the epilogue, it keeps the bias in O to a few blocks' worth, so the
    // fp32 cancellation does not grow with the partition.  Warp-uniform.
    __device__ __forceinline__ void flush_bias()
    {
        if constexpr (Codes::kBias != 0.f) {
            float b0 = ps_run0, b1 = ps_run1;
#pragma unroll
            for (int m = 4; m < 32; m <<= 1) {
                b0 += __shfl_xor_sync(kFullMask, b0, m);
                b1 += __shfl_xor_sync(kFullMask, b1, m);
            }
            b0 *= Codes::kBias;
            b1 *= Codes::kBias;
#pragma unroll
            for (int mt = 0; mt < S::MT; ++mt) {
                o[mt][0] -= b0;
                o[mt][1] -= b1;
                o[mt][2] -= b0;
                o[mt][3] -= b1;
            }
            ps_run0 = ps_run1 = 0.f;
        }
    }

    // The warp's (max, exp-sum, output) of its heads into the epilogue area.
    __device__ __forceinline__ void store(float* epi_o, float* epi_m, float* epi_l, int warp,
                                          float v_scale)
    {
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            l_run0 += __shfl_xor_sync(kFullMask, l_run0, m);
            l_run1 += __shfl_xor_sync(kFullMask, l_run1, m);
        }
        flush_bias();
        const int h0 = 2 * tig, h1 = 2 * tig + 1;
#pragma unroll
        for (int q = 0; q < S::VQ; ++q) {
            const int d = S::DPT * grp + 4 * q;
            if (h0 < G)
                *reinterpret_cast<float4*>(epi_o + (warp * G + h0) * D + d) =
                    make_float4(o[2 * q][0] * v_scale, o[2 * q][2] * v_scale,
                                o[2 * q + 1][0] * v_scale, o[2 * q + 1][2] * v_scale);
            if (h1 < G)
                *reinterpret_cast<float4*>(epi_o + (warp * G + h1) * D + d) =
                    make_float4(o[2 * q][1] * v_scale, o[2 * q][3] * v_scale,
                                o[2 * q + 1][1] * v_scale, o[2 * q + 1][3] * v_scale);
        }
        if (grp == 0) {
            if (h0 < G) {
                epi_m[warp * G + h0] = m_run0;
                epi_l[warp * G + h0] = l_run0;
            }
            if (h1 < G) {
                epi_m[warp * G + h1] = m_run1;
                epi_l[warp * G + h1] = l_run1;
            }
        }
    }
};


// One CTA: (kv head, partition, sequence).  The kernels below instantiate
// it for each code format.
template <typename Codes, typename T, int D, int BS, int G, bool ROWS>
__device__ __forceinline__ void paged_decode_q8_cta(
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
    using S = Q8Shape<D, BS, G, ROWS>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int kvh = blockIdx.x;
    const int part = blockIdx.y;
    const int s = lpt_seqs > 0
                      ? lpt_sequence(context_lens, block_tables, max_blocks_per_seq, lpt_seqs,
                                     blockIdx.z, reinterpret_cast<int32_t*>(smem))
                      : static_cast<int>(blockIdx.z);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

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
    // the block (of this partition) holding the new token, when appending
    const int append_blk = (new_key != nullptr && part == nparts - 1) ? (ctx - 1) / BS - blk_begin : -1;

    unsigned char* wbase = smem + warp * S::WARP_BYTES;
    float* wsc = reinterpret_cast<float*>(smem + S::OFF_SC) + warp * S::NSTAGE * (S::SC_STAGE / 4);
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
    auto issue = [&](int k) {
        const int chunk = k >> 5;
        if (chunk != prod_chunk) {
            prod_tbl = load_table(chunk);
            prod_chunk = chunk;
        }
        const int phys = __shfl_sync(kFullMask, prod_tbl, k & 31);
        if (warp + kWarps * k == append_blk) {
            if (phys >= 0 && static_cast<int64_t>(phys) < num_blocks) {
                if constexpr (ROWS)
                    append_row_warp_rowscale<Codes, T, D, BS>(new_key, new_value, k_cache, v_cache,
                                                              k_scales, v_scales, s, kvh,
                                                              num_kv_heads, ctx - 1, phys, lane);
                else
                    append_row_warp_q8<Codes, T, D, BS>(new_key, new_value, k_cache, v_cache, s,
                                                        kvh, num_kv_heads, ctx - 1, phys, k_inv,
                                                        v_inv, lane);
            } else if (lane == 0) {
                status_or(d_status, PA_STATUS_BAD_SLOT);
            }
        }
        if (lane == 0) {
            const int st = k % S::NSTAGE;
            const bool ok = phys >= 0 && static_cast<int64_t>(phys) < num_blocks;
            fence_proxy_async_smem();
            if (ok) {
                mbar_arrive_expect_tx(&wbar[st], 2u * S::TILE + static_cast<uint32_t>(S::SC_STAGE));
                unsigned char* dst = wbase + st * S::STAGE;
                tma_load_4d(dst, &tm_k, 0, kvh, 0, phys, &wbar[st]);
                tma_load_4d(dst + S::TILE, &tm_v, 0, kvh, 0, phys, &wbar[st]);
                if constexpr (ROWS) {
                    // the block's B row scales of this kv head: one contiguous run each
                    const int64_t so = (static_cast<int64_t>(phys) * num_kv_heads + kvh) * BS;
                    float* sc = wsc + st * (S::SC_STAGE / 4);
                    bulk_copy_g2s(sc, k_scales + so, BS * 4, &wbar[st]);
                    bulk_copy_g2s(sc + BS, v_scales + so, BS * 4, &wbar[st]);
                }
            } else {
                status_or(d_status, PA_STATUS_BAD_BLOCK);
                mbar_arrive_expect_tx(&wbar[st], 0u);
            }
        }
    };
    const int prologue = min(nk, S::NSTAGE);
    for (int k = 0; k < prologue; ++k) issue(k);
    int issued = prologue;

    Q8Warp<Codes, T, D, BS, G, ROWS> w;
    w.grp = lane >> 2;
    w.tig = lane & 3;
    w.pt_addr = smem_u32(smem + S::OFF_PT + warp * S::PT_BYTES) + (lane & 7) * S::PT_STRIDE +
                ((lane >> 3) & 1) * 16;
    w.reset();
    w.load_q(query, s, kvh, num_q_heads);

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
        const int t0 = tok_begin + (warp + kWarps * k) * BS;
        const int nv = ok ? min(BS, tok_end - t0) : 0;
        const unsigned char* kt = wbase + st * S::STAGE;
        const float* sc = wsc + st * (S::SC_STAGE / 4);
        w.block(kt, kt + S::TILE, nv, scale_log2, sc, sc + BS);
        if (k % kBiasFlushBlocks == kBiasFlushBlocks - 1) w.flush_bias();
        __syncwarp();   // every lane is done with this stage
        if (issued < nk) issue(issued++);
    }

    if (aborted) drain_after_timeout<S::NSTAGE>(wbar, first_pending, issued, d_status);

    // every warp is done with its stage buffers, unless one gave up waiting
    if (__syncthreads_or(aborted)) {
        store_aborted_rows<T, D, G>(out, ws_o, ws_ml, s, kvh, part, nparts, num_q_heads, max_parts);
        return;
    }
    float* epi_o = reinterpret_cast<float*>(smem);   // [warp][g][D]
    float* epi_m = epi_o + kWarps * G * D;
    float* epi_l = epi_m + kWarps * G;
    w.store(epi_o, epi_m, epi_l, warp, ROWS ? w.vref : v_scale);
    __syncthreads();
    merge_warps_and_store<T, D, G>(epi_o, epi_m, epi_l, out, ws_o, ws_ml, s, kvh, part, nparts,
                                   num_q_heads, max_parts);
}

#define PA_Q8_KERNEL_PARAMS                                                                     \
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,        \
        T *__restrict__ out, const T *__restrict__ query,                                      \
        const int32_t *__restrict__ block_tables, const int32_t *__restrict__ context_lens,    \
        int32_t num_q_heads, int32_t max_blocks_per_seq, int64_t num_blocks,                   \
        int32_t max_context_len, float scale_log2, float v_scale, int32_t partition_size,      \
        int32_t max_parts, float *__restrict__ ws_o, float2 *__restrict__ ws_ml,               \
        int32_t *d_status, int32_t lpt_seqs, const T *__restrict__ new_key,                    \
        const T *__restrict__ new_value, uint8_t *__restrict__ k_cache,                        \
        uint8_t *__restrict__ v_cache, int32_t num_kv_heads, float k_inv, float v_inv,          \
        uint32_t probe_us, float *__restrict__ k_scales, float *__restrict__ v_scales
#define PA_Q8_KERNEL_ARGS                                                                       \
    tm_k, tm_v, out, query, block_tables, context_lens, num_q_heads, max_blocks_per_seq,       \
        num_blocks, max_context_len, scale_log2, v_scale, partition_size, max_parts, ws_o,     \
        ws_ml, d_status, lpt_seqs, new_key, new_value, k_cache, v_cache, num_kv_heads, k_inv,  \
        v_inv, probe_us, k_scales, v_scales

// e4m3 pools (ROWS: with row-scale pools; else one scale per pool)
template <typename T, int D, int BS, int G, bool ROWS>
__global__ void __launch_bounds__(kThreads, 4) paged_decode_fp8_kernel(PA_Q8_KERNEL_PARAMS)
{
    paged_decode_q8_cta<E4m3Codes, T, D, BS, G, ROWS>(PA_Q8_KERNEL_ARGS);
}

// int8 pools
template <typename T, int D, int BS, int G, bool ROWS>
__global__ void __launch_bounds__(kThreads, 4) paged_decode_int8_kernel(PA_Q8_KERNEL_PARAMS)
{
    paged_decode_q8_cta<Int8Codes, T, D, BS, G, ROWS>(PA_Q8_KERNEL_ARGS);
}

}  // namespace pa
