// paged_decode_fp8.cuh -- decode over K/V pools stored in FP8 (e4m3) with
// per-tensor scales.  Included by paged_decode.cu.
//
// "PagedAttention：大模型KV Cache分页管理优化实践" §7 and "vLLM用虚拟内存分页思想
// 管理KV Cache" (工程实践与局限) name low-precision storage of the cached blocks;
// at one byte per element every decode step moves half the bytes.
//
// Same work split, TMA pipeline, softmax and merge as paged_decode_mma_kernel.
// Per block, the warp's K and V tiles arrive as bytes (B rows x D codes);
// the warp widens them exactly to fp16 (every e4m3 value is an fp16 value)
// into the 128-byte-swizzled 16-bit layout the tensor-core contraction reads
// with ldmatrix, clearing V rows past the context on the way.  Both
// contractions run as fp16 mma.sync with fp32 accumulation, whatever the
// query type (a bf16 query is rounded to fp16 once per CTA).  The scales are
// folded in: k_scale into the score scale, v_scale into the output.

namespace pa {

template <int D, int BS, int G>
struct Fp8Shape {
    static constexpr int NH = D / 64;
    static constexpr int KSTEPS = D / 16;
    static constexpr int NTILES = D / 8;
    static constexpr int SLICES = BS / 16;
    static constexpr int TILE8 = BS * D;                 // bytes of one K (or V) tile, one head
    static constexpr int TILE16 = BS * D * 2;            // the same tile widened to fp16
    static constexpr int STAGE8 = 2 * TILE8;
    static constexpr int NSTAGE = 2;
    static constexpr int WARP_BYTES = NSTAGE * STAGE8 + 2 * TILE16;   // byte ring + fp16 K, V
    static constexpr int OFF_BARS = kWarps * WARP_BYTES;
    static constexpr int SMEM_BYTES = OFF_BARS + kWarps * NSTAGE * 8 + 1024;
    static constexpr int EPI_BYTES = kWarps * G * (D + 2) * 4;
    static_assert(BS % 16 == 0 && D % 64 == 0, "whole 16-token slices, 128-byte rows");
    static_assert(G >= 1 && G <= 8, "heads fit rows 0..7 of the A operand");
    static_assert(EPI_BYTES <= OFF_BARS, "epilogue fits in the warp buffers");
    static_assert((NSTAGE * STAGE8) % 1024 == 0 && TILE16 % 1024 == 0,
                  "fp16 tiles keep the 1024-byte swizzle alignment");
};

// 16 e4m3 codes -> 16 fp16 values, exact.
__device__ __forceinline__ void widen16(const uint4& w, uint4& lo, uint4& hi)
{
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t r[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>(in[i] & 0xffffu), __NV_E4M3);
        const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>(in[i] >> 16), __NV_E4M3);
        r[2 * i] = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
        r[2 * i + 1] = static_cast<uint32_t>(b.x) | (static_cast<uint32_t>(b.y) << 16);
    }
    lo = make_uint4(r[0], r[1], r[2], r[3]);
    hi = make_uint4(r[4], r[5], r[6], r[7]);
}

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(kThreads, 3) paged_decode_fp8_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    T* __restrict__ out, const T* __restrict__ query, const int32_t* __restrict__ block_tables,
    const int32_t* __restrict__ context_lens, int32_t num_q_heads, int32_t max_blocks_per_seq,
    int64_t num_blocks, int32_t max_context_len, float scale_log2, float v_scale,
    int32_t partition_size, int32_t max_parts, float* __restrict__ ws_o,
    float2* __restrict__ ws_ml, int32_t* d_status)
{
    grid_dependency_wait();   // before any global access (see pa_common.cuh)
    using S = Fp8Shape<D, BS, G>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int kvh = blockIdx.x;
    const int part = blockIdx.y;
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int grp = lane >> 2;
    const int tig = lane & 3;

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

    unsigned char* wbase = smem + warp * S::WARP_BYTES;
    unsigned char* k16 = wbase + S::NSTAGE * S::STAGE8;
    unsigned char* v16 = k16 + S::TILE16;
    uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + S::OFF_BARS) + warp * S::NSTAGE;
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < S::NSTAGE; ++st) mbar_init(&wbar[st], 1);
        fence_barrier_init();
    }
    __syncwarp();

    const int32_t* table = block_tables + static_cast<int64_t>(s) * max_blocks_per_seq + blk_begin;
    auto load_table = [&](int chunk) -> int {
        const int kk = chunk * 32 + lane;
        return kk < nk ? table[warp + kWarps * kk] : -1;
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
                mbar_arrive_expect_tx(&wbar[st], 2u * S::TILE8);
                unsigned char* dst = wbase + st * S::STAGE8;
                tma_load_4d(dst, &tm_k, 0, kvh, 0, phys, &wbar[st]);
                tma_load_4d(dst + S::TILE8, &tm_v, 0, kvh, 0, phys, &wbar[st]);
            } else {
                status_or(d_status, PA_STATUS_BAD_BLOCK);
                mbar_arrive_expect_tx(&wbar[st], 0u);
            }
        }
    };
    const int prologue = min(nk, S::NSTAGE);
    for (int k = 0; k < prologue; ++k) issue(k);
    int issued = prologue;

    // q as fp16 A fragments (rows = heads; rows >= G zero)
    uint32_t qa[S::KSTEPS][2];
    {
        const T* qrow = query + (static_cast<int64_t>(s) * num_q_heads + kvh * G + grp) * D;
#pragma unroll
        for (int ks = 0; ks < S::KSTEPS; ++ks) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t packed = 0u;
                if (grp < G) {
                    const float2 f = Elem<T>::to_float2(
                        *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + half * 8 + 2 * tig));
                    packed = Elem<__half>::from_float2(f.x, f.y);
                }
                qa[ks][half] = packed;
            }
        }
    }

    const int mi = lane >> 3;
    const int ri = lane & 7;
    const uint32_t k16_base = smem_u32(k16);
    const uint32_t v16_base = smem_u32(v16);
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
        const unsigned char* k8 = wbase + st * S::STAGE8;
        const unsigned char* v8 = k8 + S::TILE8;

        // widen both tiles to fp16 in the swizzled layout; V rows past the
        // context are cleared (p = 0 does not cancel a NaN in the sum)
        for (int i = lane; i < S::TILE8 / 16; i += 32) {
            const int t = i / (D / 16);
            const int d0 = (i % (D / 16)) * 16;
            uint4 lo, hi;
            widen16(*reinterpret_cast<const uint4*>(k8 + i * 16), lo, hi);
            *reinterpret_cast<uint4*>(k16 + swz_offset<BS>(t, d0)) = lo;
            *reinterpret_cast<uint4*>(k16 + swz_offset<BS>(t, d0 + 8)) = hi;
            if (t < nv) {
                widen16(*reinterpret_cast<const uint4*>(v8 + i * 16), lo, hi);
            } else {
                lo = make_uint4(0, 0, 0, 0);
                hi = lo;
            }
            *reinterpret_cast<uint4*>(v16 + swz_offset<BS>(t, d0)) = lo;
            *reinterpret_cast<uint4*>(v16 + swz_offset<BS>(t, d0 + 8)) = hi;
        }
        __syncwarp();
        // the byte stage is free again: request the next block now
        if (issued < nk) issue(issued++);

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
                    ldmatrix_x4(b, k16_base + swz_offset<BS>(t, kp * 32 + mi * 8));
                    mma_16816<__half>(sc[nt], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, b[0], b[1]);
                    mma_16816<__half>(sc[nt], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, b[2], b[3]);
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
            for (int e = 0; e < 4; ++e) p[e] = grp < G ? exp2f(x[e] - m_sub) : 0.f;
            const uint32_t pa0 = Elem<__half>::from_float2(p[0], p[1]);
            const uint32_t pa2 = Elem<__half>::from_float2(p[2], p[3]);
            const float2 r0 = Elem<__half>::to_float2(pa0), r2 = Elem<__half>::to_float2(pa2);
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
                    ldmatrix_x4_trans(b, v16_base + swz_offset<BS>(t, np * 16 + (mi >> 1) * 8));
                    mma_16816<__half>(o[2 * np], pa0, 0u, pa2, 0u, b[0], b[1]);
                    mma_16816<__half>(o[2 * np + 1], pa0, 0u, pa2, 0u, b[2], b[3]);
                }
            }
        }
        __syncwarp();   // the fp16 tiles are rewritten by the next block
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
    float* epi_o = reinterpret_cast<float*>(smem);
    float* epi_m = epi_o + kWarps * G * D;
    float* epi_l = epi_m + kWarps * G;
    if (grp < G) {
#pragma unroll
        for (int nt = 0; nt < S::NTILES; ++nt)
            *reinterpret_cast<float2*>(epi_o + (warp * G + grp) * D + nt * 8 + 2 * tig) =
                make_float2(o[nt][0] * v_scale, o[nt][1] * v_scale);
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
