/*
 * pa_oracle.c -- plain fp64 CPU oracle for the paged-KV-cache decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library under paged_kv_cache_415_b200/) shares no code with it
 * and never calls it.
 *
 * It is deliberately slow and obvious: every output is the textbook
 * definition written out in double precision, with no blocking, fusion or
 * reordering beyond what the definition states.
 *
 * Pages cited (title, then section):
 *   [VM-paging] "vLLM用虚拟内存分页思想管理KV Cache"
 *   [Practice]  "PagedAttention：大模型KV Cache分页管理优化实践"
 *   [Manager]   "深入解析 vLLM 的 KV Cache 管理器：从内存碎片到 PagedAttention 的完整技术剖析"
 *
 * Cache layout (one layer, K and V in separate pools):
 *   k_cache, v_cache : [num_blocks][block_size][num_kv_heads][head_dim]
 * A physical block holds block_size tokens x kv heads x head_dim for K (and
 * the same for V) [Practice §3.1 物理块分配器设计].  Token t of a sequence
 * lives in logical block t / block_size at offset t % block_size, and the
 * sequence's block table maps the logical block to a physical block id
 * [Practice §3.2 块表与地址转换].
 *
 * Element storage is the raw 16-bit pattern (IEEE binary16 or bfloat16);
 * the oracle decodes the bits itself, exactly, into double.  Quantised
 * pools hold one byte per element (an e4m3 or an int8 code) and one scale
 * per pool; their functions carry the _fp8 / _int8 suffix.
 *
 * Status bits returned by the functions (same meaning as the library's):
 *   1 = a block-table entry outside [0, num_blocks)   (that block is skipped)
 *   2 = a slot at or beyond num_blocks * block_size   (that token is skipped)
 *   4 = a context length that is negative or longer than the block table
 *       (the output row is written as zeros)
 *   8 = copy_blocks: a destination written twice, or also used as a source
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_DTYPE_F16 = 0, OR_DTYPE_BF16 = 1 };

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction
 * bits.  Subnormals are fraction x 2^-24.  Every binary16 value is exact in
 * double. */
static double f16_bits_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac + 1024), expo - 25);
    return sign ? -v : v;
}

/* bfloat16: the upper half of an IEEE binary32, 8 exponent bits (bias 127),
 * 7 fraction bits.  Subnormals are fraction x 2^-133. */
static double bf16_bits_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 7) & 0xff;
    int frac = h & 0x7f;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -133);
    else if (expo == 255)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac + 128), expo - 134);
    return sign ? -v : v;
}

static double decode(uint16_t bits, int dtype)
{
    return dtype == OR_DTYPE_BF16 ? bf16_bits_to_f64(bits) : f16_bits_to_f64(bits);
}

/* Exposed so the tests can pin the bit decoding against numpy's float16 and
 * against hand-computed bfloat16 values. */
void oracle_decode_bits(const uint16_t* bits, double* out, int64_t n, int32_t dtype)
{
    for (int64_t i = 0; i < n; ++i) out[i] = decode(bits[i], dtype);
}

/* ------------------------------------------------------------------------
 * FP8 E4M3 (OCP "e4m3fn"): 1 sign bit, 4 exponent bits (bias 7), 3 fraction
 * bits, no infinities; 0x7F / 0xFF are NaN; the largest finite value is
 * 448 = 1.75 x 2^8; subnormals are fraction x 2^-9.  Cached K/V stored in
 * 8 bits with a per-tensor scale ("PagedAttention：大模型KV Cache分页管理优化实践"
 * §7: FP8/INT8 storage of history blocks; "vLLM用虚拟内存分页思想管理KV Cache",
 * 工程实践与局限: low-precision storage of block KV values).
 * ---------------------------------------------------------------------- */
static double e4m3_to_f64(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int expo = (b >> 3) & 0xf;
    int frac = b & 7;
    double v;
    if (expo == 15 && frac == 7)
        v = NAN;
    else if (expo == 0)
        v = ldexp((double)frac, -9);
    else
        v = ldexp((double)(frac + 8), expo - 10);
    return sign ? -v : v;
}

void oracle_decode_e4m3(const uint8_t* codes, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_to_f64(codes[i]);
}

/* fp32 -> e4m3, round to nearest (ties to even), values beyond the largest
 * finite magnitude saturate to +-448, NaN -> 0x7F.  Done by exact search
 * over the 126 finite non-negative codes in double: the candidates below and
 * above |x| and the tie rule decide. */
static uint8_t f32_to_e4m3(float x)
{
    if (x != x) return 0x7f;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7e);
    /* largest code with value <= a */
    int lo = 0;
    for (int c = 0; c <= 0x7e; ++c)
        if (e4m3_to_f64((uint8_t)c) <= a) lo = c;
    int hi = lo < 0x7e ? lo + 1 : lo;
    double vlo = e4m3_to_f64((uint8_t)lo), vhi = e4m3_to_f64((uint8_t)hi);
    int pick;
    if (a - vlo < vhi - a) pick = lo;
    else if (a - vlo > vhi - a) pick = hi;
    else pick = (lo & 1) ? hi : lo;        /* tie: even fraction (even code) */
    return (uint8_t)(sign | pick);
}

void oracle_encode_e4m3(const float* x, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_e4m3(x[i]);
}

/* ------------------------------------------------------------------------
 * INT8: two's-complement codes; the stored value is code x scale, one scale
 * per pool (the same passages name INT8 beside FP8).
 * ---------------------------------------------------------------------- */
static double int8_to_f64(uint8_t b)
{
    return (double)(int8_t)b;
}

void oracle_decode_int8(const uint8_t* codes, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = int8_to_f64(codes[i]);
}

/* fp32 -> int8: NaN -> 0; values at or beyond the ends of [-128, 127]
 * saturate; in-range values round to the nearest integer, ties to the even
 * one.  floor() and the fraction are exact in double. */
static uint8_t f32_to_int8(float x)
{
    if (x != x) return 0;
    if (x <= -128.0f) return (uint8_t)(int8_t)-128;
    if (x >= 127.0f) return 127;
    const double a = (double)x;
    const double lo = floor(a), frac = a - lo;
    double r;
    if (frac < 0.5) r = lo;
    else if (frac > 0.5) r = lo + 1.0;
    else r = fmod(lo, 2.0) == 0.0 ? lo : lo + 1.0;
    return (uint8_t)(int8_t)r;
}

void oracle_encode_int8(const float* x, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_int8(x[i]);
}

/* Quantising cache write: code = encode(fp32(x) * fp32(1 / scale)), the
 * product rounded once in fp32, then encoded as above (e4m3 or int8). */
static int32_t reshape_and_cache_q8(const uint16_t* key, const uint16_t* value, uint8_t* k_cache,
                                    uint8_t* v_cache, const int64_t* slot_mapping,
                                    int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t block_size, int64_t num_blocks, int32_t dtype,
                                    float k_scale, float v_scale, uint8_t (*encode)(float))
{
    int32_t status = 0;
    const float k_inv = 1.0f / k_scale, v_inv = 1.0f / v_scale;
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * (int64_t)block_size) { status |= 2; continue; }
        for (int64_t e = 0; e < row; ++e) {
            const float kx = (float)(dtype == OR_DTYPE_BF16 ? bf16_bits_to_f64(key[t * row + e])
                                                            : f16_bits_to_f64(key[t * row + e]));
            const float vx = (float)(dtype == OR_DTYPE_BF16 ? bf16_bits_to_f64(value[t * row + e])
                                                            : f16_bits_to_f64(value[t * row + e]));
            const float kq = kx * k_inv;
            const float vq = vx * v_inv;
            k_cache[slot * row + e] = encode(kq);
            v_cache[slot * row + e] = encode(vq);
        }
    }
    return status;
}

int32_t oracle_reshape_and_cache_fp8(const uint16_t* key, const uint16_t* value, uint8_t* k_cache,
                                     uint8_t* v_cache, const int64_t* slot_mapping,
                                     int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int64_t num_blocks, int32_t dtype,
                                     float k_scale, float v_scale)
{
    return reshape_and_cache_q8(key, value, k_cache, v_cache, slot_mapping, num_tokens,
                                num_kv_heads, head_dim, block_size, num_blocks, dtype, k_scale,
                                v_scale, f32_to_e4m3);
}

int32_t oracle_reshape_and_cache_int8(const uint16_t* key, const uint16_t* value,
                                      uint8_t* k_cache, uint8_t* v_cache,
                                      const int64_t* slot_mapping, int32_t num_tokens,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                      int64_t num_blocks, int32_t dtype, float k_scale,
                                      float v_scale)
{
    return reshape_and_cache_q8(key, value, k_cache, v_cache, slot_mapping, num_tokens,
                                num_kv_heads, head_dim, block_size, num_blocks, dtype, k_scale,
                                v_scale, f32_to_int8);
}

/* ------------------------------------------------------------------------
 * Row-scaled one-byte pools: every (token, kv head) row of K, and of V, has
 * a scale of its own instead of one per pool.  The scales sit in pools of
 * fp32 values beside the codes,
 *   k_scales, v_scales : [num_blocks][num_kv_heads][block_size],
 * so the cached value of element d of the row of slot `slot`, kv head g, is
 *   dec(code) * scales[slot / block_size][g][slot % block_size].
 * The pages name FP8/INT8 storage of the cached blocks ("PagedAttention：
 * 大模型KV Cache分页管理优化实践" §7, item 2; "vLLM用虚拟内存分页思想管理KV
 * Cache", 工程实践与局限) and fix no scale granularity; this is the reading
 * in which a row is quantised once, when it is written, and never again.
 *
 * The write takes each row's scale from the row itself:
 *   amax   = max_d |x_d|              (x_d: the exact fp32 value of the input)
 *   s      = fp32(amax / code_max)    (code_max 448 for e4m3, 127 for int8)
 *   code_d = encode(fp32(x_d * fp32(1 / s)))   -- the per-pool write with
 *            scale s, so the row's largest element takes the top code;
 * a row with s below the smallest normal fp32 (all zeros, or values below
 * about 1e-35) stores s = 0 and every code 0.
 * ---------------------------------------------------------------------- */
static void quantise_row(const uint16_t* x16, int32_t head_dim, int32_t dtype, float code_max,
                         uint8_t (*encode)(float), uint8_t* codes, float* scale)
{
    float amax = 0.0f;
    for (int32_t d = 0; d < head_dim; ++d) {
        const float a = fabsf((float)decode(x16[d], dtype));
        if (a > amax) amax = a;
    }
    const float s = amax / code_max;
    if (!(s >= FLT_MIN)) {
        for (int32_t d = 0; d < head_dim; ++d) codes[d] = 0;
        *scale = 0.0f;
        return;
    }
    const float inv = 1.0f / s;
    for (int32_t d = 0; d < head_dim; ++d) {
        const float x = (float)decode(x16[d], dtype);
        const float xq = x * inv;
        codes[d] = encode(xq);
    }
    *scale = s;
}

static int32_t reshape_and_cache_q8_rowscale(const uint16_t* key, const uint16_t* value,
                                             uint8_t* k_cache, uint8_t* v_cache, float* k_scales,
                                             float* v_scales, const int64_t* slot_mapping,
                                             int32_t num_tokens, int32_t num_kv_heads,
                                             int32_t head_dim, int32_t block_size,
                                             int64_t num_blocks, int32_t dtype, float code_max,
                                             uint8_t (*encode)(float))
{
    int32_t status = 0;
    for (int32_t t = 0; t < num_tokens; ++t) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * (int64_t)block_size) { status |= 2; continue; }
        const int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t g = 0; g < num_kv_heads; ++g) {
            const int64_t src = ((int64_t)t * num_kv_heads + g) * head_dim;
            const int64_t dst = (slot * num_kv_heads + g) * head_dim;
            const int64_t si = (blk * num_kv_heads + g) * block_size + off;
            quantise_row(key + src, head_dim, dtype, code_max, encode, k_cache + dst, &k_scales[si]);
            quantise_row(value + src, head_dim, dtype, code_max, encode, v_cache + dst,
                         &v_scales[si]);
        }
    }
    return status;
}

int32_t oracle_reshape_and_cache_fp8_rowscale(const uint16_t* key, const uint16_t* value,
                                              uint8_t* k_cache, uint8_t* v_cache, float* k_scales,
                                              float* v_scales, const int64_t* slot_mapping,
                                              int32_t num_tokens, int32_t num_kv_heads,
                                              int32_t head_dim, int32_t block_size,
                                              int64_t num_blocks, int32_t dtype)
{
    return reshape_and_cache_q8_rowscale(key, value, k_cache, v_cache, k_scales, v_scales,
                                         slot_mapping, num_tokens, num_kv_heads, head_dim,
                                         block_size, num_blocks, dtype, 448.0f, f32_to_e4m3);
}

int32_t oracle_reshape_and_cache_int8_rowscale(const uint16_t* key, const uint16_t* value,
                                               uint8_t* k_cache, uint8_t* v_cache,
                                               float* k_scales, float* v_scales,
                                               const int64_t* slot_mapping, int32_t num_tokens,
                                               int32_t num_kv_heads, int32_t head_dim,
                                               int32_t block_size, int64_t num_blocks,
                                               int32_t dtype)
{
    return reshape_and_cache_q8_rowscale(key, value, k_cache, v_cache, k_scales, v_scales,
                                         slot_mapping, num_tokens, num_kv_heads, head_dim,
                                         block_size, num_blocks, dtype, 127.0f, f32_to_int8);
}

/* ------------------------------------------------------------------------
 * reshape_and_cache: write each new token's K and V rows into the slot the
 * allocator gave it ([Practice §3.3 按需分配策略], step 4 "write the new
 * token's KV vectors"; [Manager, 第一部分 KV Cache 的核心价值]: the new K/V is
 * appended before attention).  slot = physical_block * block_size + offset.
 * A negative slot is a padding token and writes nothing.  It is a raw bit
 * copy: no value changes.
 * ---------------------------------------------------------------------- */
int32_t oracle_reshape_and_cache(const uint16_t* key, const uint16_t* value,
                                 uint16_t* k_cache, uint16_t* v_cache,
                                 const int64_t* slot_mapping, int32_t num_tokens,
                                 int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int64_t num_blocks)
{
    int32_t status = 0;
    const int64_t row = (int64_t)num_kv_heads * head_dim; /* elements per token */
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * (int64_t)block_size) { status |= 2; continue; }
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            for (int32_t d = 0; d < head_dim; ++d) {
                int64_t src = (int64_t)t * row + (int64_t)h * head_dim + d;
                int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * head_dim + d;
                k_cache[dst] = key[src];
                v_cache[dst] = value[src];
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------------
 * copy_blocks: the data half of copy-on-write.  When a sequence must modify
 * a block whose reference count is above one, the manager allocates a new
 * block, copies the original's data into it, remaps privately and drops the
 * old reference ([VM-paging, 写时复制与块共享机制]; [Practice §4.1 共享内存管理]
 * steps 1-4).  This is step 2, for every (src, dst) pair, in order, for K
 * and V.  src == dst is a no-op.  A destination that appears twice, or that
 * is also a source in the same call, raises status bit 8 (the pairs are
 * still applied in order here).
 * ---------------------------------------------------------------------- */
int32_t oracle_copy_blocks(uint16_t* k_cache, uint16_t* v_cache,
                           const int64_t* block_mapping, int32_t num_pairs,
                           int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int64_t num_blocks)
{
    int32_t status = 0;
    const int64_t block_elems = (int64_t)block_size * num_kv_heads * head_dim;
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t dst = block_mapping[2 * i + 1];
        for (int32_t j = 0; j < num_pairs; ++j) {
            if (j == i) continue;
            if (block_mapping[2 * j + 1] == dst && j < i) status |= 8;
            if (block_mapping[2 * j] == dst && block_mapping[2 * j] != block_mapping[2 * j + 1])
                status |= 8;
        }
    }
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i];
        int64_t dst = block_mapping[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) { status |= 1; continue; }
        if (src == dst) continue;
        for (int64_t e = 0; e < block_elems; ++e) {
            k_cache[dst * block_elems + e] = k_cache[src * block_elems + e];
            v_cache[dst * block_elems + e] = v_cache[src * block_elems + e];
        }
    }
    return status;
}

/* ------------------------------------------------------------------------
 * swap_blocks: eviction of a waiting request's blocks to CPU memory and
 * their return when it is rescheduled ([VM-paging, 显存管理与调度策略设计],
 * the eviction paragraph).  For every (src, dst) pair, in order, block src of
 * the source pools becomes block dst of the destination pools, K and V, as
 * raw bytes (elem_bytes per element).  An id outside its own pool raises bit
 * 1 and the pair is skipped; a destination that appears twice raises bit 8
 * (the pairs are still applied in order here).
 * ---------------------------------------------------------------------- */
int32_t oracle_swap_blocks(const uint8_t* src_k, const uint8_t* src_v, uint8_t* dst_k,
                           uint8_t* dst_v, const int64_t* block_mapping, int32_t num_pairs,
                           int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                           int64_t src_num_blocks, int64_t dst_num_blocks, int32_t elem_bytes)
{
    int32_t status = 0;
    const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim * elem_bytes;
    for (int32_t i = 0; i < num_pairs; ++i)
        for (int32_t j = 0; j < i; ++j)
            if (block_mapping[2 * j + 1] == block_mapping[2 * i + 1]) status |= 8;
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i];
        int64_t dst = block_mapping[2 * i + 1];
        if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
            status |= 1;
            continue;
        }
        for (int64_t b = 0; b < block_bytes; ++b) {
            dst_k[dst * block_bytes + b] = src_k[src * block_bytes + b];
            dst_v[dst * block_bytes + b] = src_v[src * block_bytes + b];
        }
    }
    return status;
}

/* Address translation: token t of sequence s -> element offset of row
 * (t, kv head g) in the pool, or -1 when the table entry is out of range
 * ([Practice §3.2]: logical block j -> table[j] -> physical id -> base +
 * offset). */
static int64_t token_row(const int32_t* table, int32_t t, int32_t g,
                         int32_t num_kv_heads, int32_t head_dim,
                         int32_t block_size, int64_t num_blocks)
{
    int64_t phys = table[t / block_size];
    if (phys < 0 || phys >= num_blocks) return -1;
    return ((phys * block_size + t % block_size) * num_kv_heads + g) * (int64_t)head_dim;
}

/* ------------------------------------------------------------------------
 * Paged decode attention for one (sequence, query head), direct form.
 *
 * [VM-paging, PagedAttention的注意力计算流程]: for request i and head l, take
 * the physical blocks from the block table; pass 1 scores the query against
 * every Key in those blocks; softmax gives the weights; pass 2 sums the
 * Values with those weights.  [Manager, 第二部分 PagedAttention 的核心思想]
 * step 4: the kernel reassembles K/V through the block table at run time.
 *
 * Query head h reads kv head h / (num_q_heads / num_kv_heads) (consecutive
 * grouping; with equal head counts this is plain multi-head attention).
 *
 *   x_t = scale * sum_d q[d] * K_t[d]          t < context_len
 *   w_t = exp(x_t - max x) / sum_u exp(x_u - max x)
 *   out = sum_t w_t * V_t
 * ---------------------------------------------------------------------- */
static int32_t decode_row(double* out, const uint16_t* query, const uint16_t* k_cache,
                          const uint16_t* v_cache, const int32_t* block_tables,
                          const int32_t* context_lens, int32_t s, int32_t h,
                          int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t block_size, int32_t max_blocks_per_seq,
                          int64_t num_blocks, double scale, int32_t dtype,
                          int32_t blocked)
{
    int32_t status = 0;
    const int32_t group = num_q_heads / num_kv_heads;
    const int32_t g = h / group;
    const int32_t ctx = context_lens[s];
    const int32_t* table = block_tables + (int64_t)s * max_blocks_per_seq;
    for (int32_t d = 0; d < head_dim; ++d) out[d] = 0.0;
    if (ctx < 0 || ctx > (int64_t)max_blocks_per_seq * block_size) return 4;
    if (ctx == 0) return 0;

    double* q = (double*)malloc(sizeof(double) * head_dim);
    double* x = (double*)malloc(sizeof(double) * ctx);
    unsigned char* valid = (unsigned char*)malloc(ctx);
    const uint16_t* qbits = query + ((int64_t)s * num_q_heads + h) * head_dim;
    for (int32_t d = 0; d < head_dim; ++d) q[d] = decode(qbits[d], dtype);

    /* pass 1: scores */
    int32_t any = 0;
    for (int32_t t = 0; t < ctx; ++t) {
        int64_t r = token_row(table, t, g, num_kv_heads, head_dim, block_size, num_blocks);
        valid[t] = r >= 0;
        if (r < 0) { status |= 1; x[t] = 0.0; continue; }
        double acc = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) acc += q[d] * decode(k_cache[r + d], dtype);
        x[t] = scale * acc;
        any = 1;
    }

    if (any) {
        double m = -INFINITY, l = 0.0;
        if (!blocked) {
            /* softmax, direct */
            for (int32_t t = 0; t < ctx; ++t) if (valid[t] && x[t] > m) m = x[t];
        } else {
            /* the five steps of [Practice §5.1 分块Softmax算法]:
             * (1) local max m_j of every block j, (2) global max over the
             * m_j, (3) the exps exp(s - m_global), (4) their global sum,
             * (5) w = exp(s - m_global) / l_global.  Steps 3-5 are shared
             * with the direct form below; steps 1-2 differ. */
            int32_t nb = (ctx + block_size - 1) / block_size;
            for (int32_t j = 0; j < nb; ++j) {
                double mj = -INFINITY;
                for (int32_t t = j * block_size; t < ctx && t < (j + 1) * block_size; ++t)
                    if (valid[t] && x[t] > mj) mj = x[t];
                if (mj > m) m = mj;
            }
        }
        for (int32_t t = 0; t < ctx; ++t) if (valid[t]) l += exp(x[t] - m);
        /* pass 2: weighted sum of Values */
        for (int32_t t = 0; t < ctx; ++t) {
            if (!valid[t]) continue;
            double w = exp(x[t] - m) / l;
            int64_t r = token_row(table, t, g, num_kv_heads, head_dim, block_size, num_blocks);
            for (int32_t d = 0; d < head_dim; ++d) out[d] += w * decode(v_cache[r + d], dtype);
        }
    }
    free(q); free(x); free(valid);
    return status;
}

/* The scale of the row at element offset r of a row-scaled pool: row
 * r / head_dim is slot * num_kv_heads + g, and its scale sits at
 * [slot / block_size][g][slot % block_size] of the scale pool. */
static double row_scale(const float* scales, int64_t r, int32_t num_kv_heads, int32_t head_dim,
                        int32_t block_size)
{
    const int64_t row = r / head_dim;
    const int64_t slot = row / num_kv_heads, g = row % num_kv_heads;
    return (double)scales[((slot / block_size) * num_kv_heads + g) * block_size + slot % block_size];
}

/* Paged decode over 8-bit pools (e4m3 or int8 codes): every cached element
 * is dequantised, K = dec(code) * k_scale, V = dec(code) * v_scale, in
 * double, and the attention is the direct form of decode_row.  Query and
 * output as in oracle_paged_decode (query bits of `dtype`).  With row-scale
 * pools (k_scales / v_scales not NULL) each row's own scale replaces the
 * pool's. */
static int32_t decode_row_q8(double* out, const uint16_t* query, const uint8_t* k_cache,
                             const uint8_t* v_cache, const int32_t* block_tables,
                             const int32_t* context_lens, int32_t s, int32_t h,
                             int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                             int32_t block_size, int32_t max_blocks_per_seq, int64_t num_blocks,
                             double scale, int32_t dtype, double k_scale, double v_scale,
                             const float* k_scales, const float* v_scales,
                             double (*dec)(uint8_t))
{
    int32_t status = 0;
    const int32_t group = num_q_heads / num_kv_heads;
    const int32_t g = h / group;
    const int32_t ctx = context_lens[s];
    const int32_t* table = block_tables + (int64_t)s * max_blocks_per_seq;
    for (int32_t d = 0; d < head_dim; ++d) out[d] = 0.0;
    if (ctx < 0 || ctx > (int64_t)max_blocks_per_seq * block_size) return 4;
    if (ctx == 0) return 0;
    double* q = (double*)malloc(sizeof(double) * head_dim);
    double* x = (double*)malloc(sizeof(double) * ctx);
    unsigned char* valid = (unsigned char*)malloc(ctx);
    const uint16_t* qbits = query + ((int64_t)s * num_q_heads + h) * head_dim;
    for (int32_t d = 0; d < head_dim; ++d) q[d] = decode(qbits[d], dtype);
    int32_t any = 0;
    for (int32_t t = 0; t < ctx; ++t) {
        int64_t r = token_row(table, t, g, num_kv_heads, head_dim, block_size, num_blocks);
        valid[t] = r >= 0;
        if (r < 0) { status |= 1; x[t] = 0.0; continue; }
        const double ks = k_scales ? row_scale(k_scales, r, num_kv_heads, head_dim, block_size)
                                   : k_scale;
        double acc = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) acc += q[d] * (dec(k_cache[r + d]) * ks);
        x[t] = scale * acc;
        any = 1;
    }
    if (any) {
        double m = -INFINITY, l = 0.0;
        for (int32_t t = 0; t < ctx; ++t) if (valid[t] && x[t] > m) m = x[t];
        for (int32_t t = 0; t < ctx; ++t) if (valid[t]) l += exp(x[t] - m);
        for (int32_t t = 0; t < ctx; ++t) {
            if (!valid[t]) continue;
            double w = exp(x[t] - m) / l;
            int64_t r = token_row(table, t, g, num_kv_heads, head_dim, block_size, num_blocks);
            const double vs = v_scales ? row_scale(v_scales, r, num_kv_heads, head_dim, block_size)
                                       : v_scale;
            for (int32_t d = 0; d < head_dim; ++d)
                out[d] += w * (dec(v_cache[r + d]) * vs);
        }
    }
    free(q); free(x); free(valid);
    return status;
}

static void set_threads(int32_t num_threads)
{
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
}

/* Full output: out is double [num_seqs][num_q_heads][head_dim]. */
int32_t oracle_paged_decode(double* out, const uint16_t* query, const uint16_t* k_cache,
                            const uint16_t* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, int32_t num_seqs,
                            int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                            int32_t block_size, int32_t max_blocks_per_seq,
                            int64_t num_blocks, double scale, int32_t dtype,
                            int32_t blocked, int32_t num_threads)
{
    int32_t status = 0;
    const int64_t rows = (int64_t)num_seqs * num_q_heads;
    set_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : status)
    for (int64_t r = 0; r < rows; ++r) {
        int32_t s = (int32_t)(r / num_q_heads), h = (int32_t)(r % num_q_heads);
        status |= decode_row(out + r * head_dim, query, k_cache, v_cache, block_tables,
                             context_lens, s, h, num_q_heads, num_kv_heads, head_dim,
                             block_size, max_blocks_per_seq, num_blocks, scale, dtype, blocked);
    }
    return status;
}

/* Selected rows only: rows is int32 [n_rows][2] of (sequence, query head);
 * out is double [n_rows][head_dim].  Used to check full-size launches on a
 * sample of outputs. */
int32_t oracle_paged_decode_rows(double* out, const int32_t* rows, int32_t n_rows,
                                 const uint16_t* query, const uint16_t* k_cache,
                                 const uint16_t* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int32_t max_blocks_per_seq, int64_t num_blocks, double scale,
                                 int32_t dtype, int32_t num_threads)
{
    int32_t status = 0;
    set_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : status)
    for (int32_t i = 0; i < n_rows; ++i) {
        status |= decode_row(out + (int64_t)i * head_dim, query, k_cache, v_cache, block_tables,
                             context_lens, rows[2 * i], rows[2 * i + 1], num_q_heads,
                             num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                             scale, dtype, 0);
    }
    return status;
}

int32_t oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int32_t paged_decode_q8(double* out, const uint16_t* query, const uint8_t* k_cache,
                               const uint8_t* v_cache, const int32_t* block_tables,
                               const int32_t* context_lens, int32_t num_seqs,
                               int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                               int32_t block_size, int32_t max_blocks_per_seq,
                               int64_t num_blocks, double scale, int32_t dtype, double k_scale,
                               double v_scale, const float* k_scales, const float* v_scales,
                               int32_t num_threads, double (*dec)(uint8_t))
{
    int32_t status = 0;
    const int64_t rows = (int64_t)num_seqs * num_q_heads;
    set_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : status)
    for (int64_t r = 0; r < rows; ++r) {
        int32_t s = (int32_t)(r / num_q_heads), h = (int32_t)(r % num_q_heads);
        status |= decode_row_q8(out + r * head_dim, query, k_cache, v_cache, block_tables,
                                context_lens, s, h, num_q_heads, num_kv_heads, head_dim,
                                block_size, max_blocks_per_seq, num_blocks, scale, dtype,
                                k_scale, v_scale, k_scales, v_scales, dec);
    }
    return status;
}

int32_t oracle_paged_decode_fp8(double* out, const uint16_t* query, const uint8_t* k_cache,
                                const uint8_t* v_cache, const int32_t* block_tables,
                                const int32_t* context_lens, int32_t num_seqs,
                                int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_blocks_per_seq,
                                int64_t num_blocks, double scale, int32_t dtype, double k_scale,
                                double v_scale, int32_t num_threads)
{
    return paged_decode_q8(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, scale, dtype, k_scale, v_scale, NULL, NULL, num_threads,
                           e4m3_to_f64);
}

int32_t oracle_paged_decode_int8(double* out, const uint16_t* query, const uint8_t* k_cache,
                                 const uint8_t* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int32_t num_seqs,
                                 int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int32_t max_blocks_per_seq,
                                 int64_t num_blocks, double scale, int32_t dtype, double k_scale,
                                 double v_scale, int32_t num_threads)
{
    return paged_decode_q8(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, scale, dtype, k_scale, v_scale, NULL, NULL, num_threads,
                           int8_to_f64);
}

/* Paged decode over row-scaled one-byte pools (scale pools as for the
 * _rowscale write above): each cached row dequantised with its own scale. */
int32_t oracle_paged_decode_fp8_rowscale(double* out, const uint16_t* query,
                                         const uint8_t* k_cache, const uint8_t* v_cache,
                                         const float* k_scales, const float* v_scales,
                                         const int32_t* block_tables, const int32_t* context_lens,
                                         int32_t num_seqs, int32_t num_q_heads,
                                         int32_t num_kv_heads, int32_t head_dim,
                                         int32_t block_size, int32_t max_blocks_per_seq,
                                         int64_t num_blocks, double scale, int32_t dtype,
                                         int32_t num_threads)
{
    return paged_decode_q8(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, scale, dtype, 1.0, 1.0, k_scales, v_scales, num_threads,
                           e4m3_to_f64);
}

int32_t oracle_paged_decode_int8_rowscale(double* out, const uint16_t* query,
                                          const uint8_t* k_cache, const uint8_t* v_cache,
                                          const float* k_scales, const float* v_scales,
                                          const int32_t* block_tables, const int32_t* context_lens,
                                          int32_t num_seqs, int32_t num_q_heads,
                                          int32_t num_kv_heads, int32_t head_dim,
                                          int32_t block_size, int32_t max_blocks_per_seq,
                                          int64_t num_blocks, double scale, int32_t dtype,
                                          int32_t num_threads)
{
    return paged_decode_q8(out, query, k_cache, v_cache, block_tables, context_lens, num_seqs,
                           num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, scale, dtype, 1.0, 1.0, k_scales, v_scales, num_threads,
                           int8_to_f64);
}
