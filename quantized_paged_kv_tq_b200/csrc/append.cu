// KV-cache writers: TurboQuant quantise-and-append, and the plain bf16 append.
//
// "xInfer: Pure-Rust LLM Inference Without a Python Runtime", section "What
// actually sits between the request and the tokens": each new K/V head
// vector is rotated by a Walsh-Hadamard transform and then absmax-quantised
// per head.  One warp handles one (token, kv head, K-or-V) vector of 128
// values: lane l holds elements 4l..4l+3, the two low butterfly stages run in
// registers, the five high stages across lanes with shuffles; the absmax is a
// warp max-reduction; codes are packed LSB-first and written with 128-bit
// stores.  Every floating-point step is an explicitly rounded fp32 operation
// (this file is compiled with -fmad=false), in the same stage order as the
// definition, so codes and scales are bit-exact.
#include <cstdint>

#include "tq_device.cuh"

namespace tq {

namespace {

constexpr int kAppendWarps = 8;

__device__ __forceinline__ void fwht128_lane(float x[4], int lane)
{
    // strides 1 and 2: inside the lane (elements 4l .. 4l+3)
    float a0 = __fadd_rn(x[0], x[1]), a1 = __fsub_rn(x[0], x[1]);
    float a2 = __fadd_rn(x[2], x[3]), a3 = __fsub_rn(x[2], x[3]);
    x[0] = __fadd_rn(a0, a2);
    x[2] = __fsub_rn(a0, a2);
    x[1] = __fadd_rn(a1, a3);
    x[3] = __fsub_rn(a1, a3);
    // strides 4 .. 64: partner lane = lane ^ (stride / 4)
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float p = __shfl_xor_sync(kFull, x[e], m);
            // lower element: a + b; upper element: a - b with a the lower one
            x[e] = upper ? __fsub_rn(p, x[e]) : __fadd_rn(x[e], p);
        }
    }
}

template <int BITS>
__device__ __forceinline__ void store_codes(uint8_t* dst, const uint32_t u[4], int lane, int sw)
{
    // the lane holding chunk c stores it at chunk c ^ sw (sw = 0 for 3 bits)
    // piece = this lane's 4 codes, LSB-first: code e at bits [e*BITS, (e+1)*BITS)
    uint32_t piece = u[0] | (u[1] << BITS) | (u[2] << (2 * BITS)) | (u[3] << (3 * BITS));
    if constexpr (BITS == 8) {
        // 32 words (128 B); chunk c = words 4c..4c+3 held by lanes 4c..4c+3
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = __shfl_sync(kFull, piece, 4 * (lane & 7) + k);
        if (lane < 8)
            *reinterpret_cast<uint4*>(dst + 16 * (lane ^ sw)) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if constexpr (BITS == 4) {
        uint32_t nb = __shfl_down_sync(kFull, piece, 1);
        uint32_t word = piece | (nb << 16);          // valid on even lanes: word lane/2
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = __shfl_sync(kFull, word, 8 * (lane & 3) + 2 * k);
        if (lane < 4)
            *reinterpret_cast<uint4*>(dst + 16 * (lane ^ sw)) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if constexpr (BITS == 2) {
        uint32_t half = piece | (__shfl_down_sync(kFull, piece, 1) << 8);
        uint32_t word = half | (__shfl_down_sync(kFull, half, 2) << 16);  // lanes 4w
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = __shfl_sync(kFull, word, 16 * (lane & 1) + 4 * k);
        if (lane < 2)
            *reinterpret_cast<uint4*>(dst + 16 * (lane ^ sw)) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {  // BITS == 3: 12-bit pieces, 48 bytes per vector
        // 24-bit groups (8 codes) on even lanes: group lane/2 at bit 24*(lane/2)
        uint32_t grp = piece | (__shfl_down_sync(kFull, piece, 1) << 12);
        // lane q < 4 assembles words 3q..3q+2 from groups 4q..4q+3
        uint32_t A = __shfl_sync(kFull, grp, 8 * (lane & 3) + 0);
        uint32_t B = __shfl_sync(kFull, grp, 8 * (lane & 3) + 2);
        uint32_t C = __shfl_sync(kFull, grp, 8 * (lane & 3) + 4);
        uint32_t D = __shfl_sync(kFull, grp, 8 * (lane & 3) + 6);
        uint32_t w0 = A | (B << 24);
        uint32_t w1 = (B >> 8) | (C << 16);
        uint32_t w2 = (C >> 16) | (D << 8);
        // lane c < 3 stores chunk c = words 4c..4c+3; word w sits in lane w/3,
        // register w%3
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int wi = 4 * (lane % 3) + k;
            const int src = wi / 3, r = wi % 3;
            uint32_t r0 = __shfl_sync(kFull, w0, src);
            uint32_t r1 = __shfl_sync(kFull, w1, src);
            uint32_t r2 = __shfl_sync(kFull, w2, src);
            w[k] = r == 0 ? r0 : (r == 1 ? r1 : r2);
        }
        if (lane < 3)
            *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Dim-major V rows: dimension i's row holds page_size fields of BITS bits,
// token t at bits [t*BITS, (t+1)*BITS).  Tokens of one page may be appended
// concurrently, so sub-byte fields are written with 32-bit atomic and/or
// (each field is owned by one token; the other bits are left alone).
template <int BITS>
__device__ __forceinline__ void store_dim_major(uint8_t* blk, const uint32_t u[4], int lane,
                                                int off, int page_size)
{
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int i = 4 * lane + e;
        const int64_t bit = (int64_t)i * page_size * BITS + (int64_t)off * BITS;
        if constexpr (BITS == 8) {
            blk[bit >> 3] = (uint8_t)u[e];
        } else {
            unsigned* w = reinterpret_cast<unsigned*>(blk) + (bit >> 5);
            const int sh = (int)(bit & 31);
            const unsigned field = (1u << BITS) - 1u;
            atomicAnd(w, ~(field << sh));
            atomicOr(w, u[e] << sh);
            if (sh + BITS > 32) {            // a 3-bit field across two words
                const int rest = sh + BITS - 32;
                atomicAnd(w + 1, ~((1u << rest) - 1u));
                atomicOr(w + 1, u[e] >> (BITS - rest));
            }
        }
    }
}

template <int BITS>
__global__ void __launch_bounds__(32 * kAppendWarps)
k_quantize_append(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                  const int64_t* __restrict__ slots, int num_tokens, int num_kv_heads,
                  int page_size, int num_pages, int64_t block_bytes,
                  uint8_t* __restrict__ pool, uint32_t* err)
{
    constexpr int L = (1 << (BITS - 1)) - 1;
    constexpr int CB = kHeadDim * BITS / 8;   // code bytes per row
    const int lane = threadIdx.x & 31;
    const int64_t vec = (int64_t)blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    const int per_tok = 2 * num_kv_heads;
    if (vec >= (int64_t)num_tokens * per_tok) return;
    const int64_t tok = vec / per_tok;
    const int r = (int)(vec - tok * per_tok);
    const int which = r >= num_kv_heads;          // 0: K, 1: V
    const int head = r - which * num_kv_heads;

    const int64_t slot = slots[tok];
    if (slot < 0) return;
    const int64_t page = slot / page_size;
    const int off = (int)(slot - page * page_size);
    if (page >= num_pages) {
        if (lane == 0) report_error(err, TQ_ERR_DEVICE_CHECK, kErrSlotRange);
        return;
    }

    const uint16_t* src = (which ? v : k) + (tok * num_kv_heads + head) * kHeadDim;
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src) + lane);
    float x[4] = {bf16_bits_to_float(raw.x & 0xffffu), bf16_bits_to_float(raw.x >> 16),
                  bf16_bits_to_float(raw.y & 0xffffu), bf16_bits_to_float(raw.y >> 16)};

    fwht128_lane(x, lane);
    const float c = __uint_as_float(0x3DB504F3u);   // fp32(1 / sqrt(128))
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[e] = __fmul_rn(x[e], c);
        amax = fmaxf(amax, fabsf(x[e]));
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, m));
    const float s = amax;

    uint32_t u[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        int code = 0;
        if (s != 0.f) {
            float q = roundf(__fdiv_rn(__fmul_rn(x[e], (float)L), s));
            q = fminf(fmaxf(q, -(float)L), (float)L);
            code = (int)q;
        }
        u[e] = (uint32_t)(code + L);
    }

    // pool[page][head][K block, V block]
    uint8_t* blk = pool + ((page * num_kv_heads + head) * 2 + which) * block_bytes;
    if (!which) {
        // K: the packed vector is token row `off`
        store_codes<BITS>(blk + (int64_t)off * CB, u, lane, k_swizzle<BITS>(off));
    } else {
        // V: dim-major rows; code i is field `off` of row i
        store_dim_major<BITS>(blk, u, lane, off, page_size);
    }
    if (lane == 0)
        *reinterpret_cast<float*>(blk + (int64_t)page_size * CB + 4 * off) = s;
}

__global__ void __launch_bounds__(32 * kAppendWarps)
k_append_bf16(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
              const int64_t* __restrict__ slots, int num_tokens, int num_kv_heads,
              int page_size, int num_pages, uint16_t* __restrict__ pool, uint32_t* err)
{
    const int lane = threadIdx.x & 31;
    const int64_t vec = (int64_t)blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    const int per_tok = 2 * num_kv_heads;
    if (vec >= (int64_t)num_tokens * per_tok) return;
    const int64_t tok = vec / per_tok;
    const int r = (int)(vec - tok * per_tok);
    const int which = r >= num_kv_heads;
    const int head = r - which * num_kv_heads;
    const int64_t slot = slots[tok];
    if (slot < 0) return;
    const int64_t page = slot / page_size;
    const int off = (int)(slot - page * page_size);
    if (page >= num_pages) {
        if (lane == 0) report_error(err, TQ_ERR_DEVICE_CHECK, kErrSlotRange);
        return;
    }
    const uint16_t* src = (which ? v : k) + (tok * num_kv_heads + head) * kHeadDim;
    uint16_t* dst = pool + ((((page * num_kv_heads + head) * 2 + which) * page_size + off) *
                            kHeadDim);
    reinterpret_cast<uint2*>(dst)[lane] = __ldg(reinterpret_cast<const uint2*>(src) + lane);
}

}  // namespace

cudaError_t launch_quantize_append(const void* k, const void* v, const int64_t* slots,
                                   int num_tokens, int bits, const tq_cache& c,
                                   int64_t block_bytes, cudaStream_t stream)
{
    const int64_t vecs = (int64_t)num_tokens * 2 * c.num_kv_heads;
    const unsigned grid = (unsigned)((vecs + kAppendWarps - 1) / kAppendWarps);
    const auto* kk = static_cast<const uint16_t*>(k);
    const auto* vv = static_cast<const uint16_t*>(v);
    auto* pool = static_cast<uint8_t*>(c.pages);
#define TQ_LAUNCH_QA(B)                                                               \
    k_quantize_append<B><<<grid, 32 * kAppendWarps, 0, stream>>>(                     \
        kk, vv, slots, num_tokens, c.num_kv_heads, c.page_size, c.num_pages,         \
        block_bytes, pool, c.dev_error)
    switch (bits) {
    case 2: TQ_LAUNCH_QA(2); break;
    case 3: TQ_LAUNCH_QA(3); break;
    case 4: TQ_LAUNCH_QA(4); break;
    case 8: TQ_LAUNCH_QA(8); break;
    default: return cudaErrorInvalidValue;
    }
#undef TQ_LAUNCH_QA
    return cudaGetLastError();
}

cudaError_t launch_append_bf16(const void* k, const void* v, const int64_t* slots,
                               int num_tokens, const tq_cache& c, cudaStream_t stream)
{
    const int64_t vecs = (int64_t)num_tokens * 2 * c.num_kv_heads;
    const unsigned grid = (unsigned)((vecs + kAppendWarps - 1) / kAppendWarps);
    k_append_bf16<<<grid, 32 * kAppendWarps, 0, stream>>>(
        static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), slots, num_tokens,
        c.num_kv_heads, c.page_size, c.num_pages, static_cast<uint16_t*>(c.pages), c.dev_error);
    return cudaGetLastError();
}

}  // namespace tq
