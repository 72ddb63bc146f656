// KV-cache writers: TurboQuant quantise-and-append, and the plain bf16 append.
//
// "xInfer: Pure-Rust LLM Inference Without a Python Runtime", section "What
// actually sits between the request and the tokens": each new K/V head
// vector is rotated by a Walsh-Hadamard transform and then absmax-quantised
// per head.  The quantiser (k_quantize_append, described below) gives each
// vector four threads and each CTA a window of tokens of one kv head, so
// that whole pages of dim-major V rows are written with 128-bit stores.
// Every floating-point step is an explicitly rounded fp32 operation (this
// file is compiled with -fmad=false; the packed fp32x2 operations round each
// lane like the scalar ones), in the same stage order as the definition, so
// codes and scales are bit-exact.
#include <cstdint>

#include "tq_device.cuh"

namespace tq {

namespace {

constexpr int kAppendWarps = 8;         // bf16 append: one warp per (token, head, K or V)

// ===================================================================
// Windowed quantise-and-append.
//
// One CTA (256 threads) owns a window of consecutive tokens of the call for
// one kv head.  Window boundaries are moved forward to the next token that
// does not continue a run (a run: tokens whose slots are consecutive inside
// one page), so a page filled in order by one call is never split between
// two CTAs.  Four threads handle one 128-value vector (thread q holds values
// 32q .. 32q + 31): the butterflies of strides 1-16 run in registers (packed
// fp32 pairs, each lane rounded like a scalar fp32 operation), those of
// strides 32 and 64 between the four threads with shuffles.  K codes are
// packed and stored as whole row pieces; V codes are staged in shared memory
// dimension-major and written as whole dim-major rows, with plain vector
// stores where the window owns every field of a word and atomic and/or only
// for words shared with tokens outside the window.
// ===================================================================
constexpr int kQaThreads = 256;
constexpr int kQaWin = 64;             // tokens per window before alignment (large calls)
constexpr int kQaMaxWin = 128;         // staging capacity: kQaWin + page_size - 1 <= 127
constexpr int kQaPass = 32;            // tokens per pass (x K and V = 64 vectors)
// staging row: window tokens (< 128, XOR 8 (dim / 32) stays below 128) and
// 8 bytes of pitch so that the V writer's 8-byte reads of rows 2 apart
// spread over the banks; two buffers, so that the writer of one head runs
// while the next head is quantised
constexpr int kVRow = 136;
constexpr int kQaStages = 2;           // input ring: each thread's next pass, by cp.async
constexpr int kQaInBytes = kQaStages * kQaThreads * 64;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                 :: "r"(smem_addr(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ unsigned long long pk2(float a, float b)
{
    unsigned long long d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ void up2(unsigned long long v, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long sub2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// x * s + p, rounded once: with s = +-1 the product is exact, so this is the
// IEEE sum p + x or difference p - x
__device__ __forceinline__ unsigned long long fma2(unsigned long long x, unsigned long long s,
                                                   unsigned long long p)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(x), "l"(s), "l"(p));
    return d;
}

// Butterflies of strides 1, 2, 4, 8, 16 over this thread's 32 values, in
// that order; x[i] holds value 32q + i.
__device__ __forceinline__ void fwht32_in_thread(float x[32])
{
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        const float a = x[i], b = x[i + 1];
        x[i] = __fadd_rn(a, b);
        x[i + 1] = __fsub_rn(a, b);
    }
#pragma unroll
    for (int h = 2; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            if (i & h) continue;
            const unsigned long long lo = pk2(x[i], x[i + 1]);
            const unsigned long long hi = pk2(x[i + h], x[i + h + 1]);
            up2(add2(lo, hi), x[i], x[i + 1]);
            up2(sub2(lo, hi), x[i + h], x[i + h + 1]);
        }
    }
}

// Strides 32 and 64: partner thread q ^ 1, then q ^ 2 (lane bits 0 and 1).
// The lower index keeps a + b, the upper one a - b (a the lower value).
__device__ __forceinline__ void fwht32_across(float x[32], int q)
{
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
        const float sg = (q & m) ? -1.f : 1.f;
        const unsigned long long sg2 = pk2(sg, sg);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const float p0 = __shfl_xor_sync(kFull, x[i], m);
            const float p1 = __shfl_xor_sync(kFull, x[i + 1], m);
            up2(fma2(pk2(x[i], x[i + 1]), sg2, pk2(p0, p1)), x[i], x[i + 1]);
        }
    }
}

// Smallest power of two >= 4 L, times 2^-24: the fast path's margin.
__host__ __device__ constexpr float quant_margin(int L)
{
    float m = 1.f / 16777216.f;
    for (int p = 1; p < 4 * L; p *= 2) m *= 2.f;
    return m;
}

// Codes of this thread's 32 rotated values y (scale s): offset-binary
// u = code + L with code = clamp(roundf(fl(y L) / s), -L, L), the division
// an IEEE fp32 one.  Fast path: with t = fl(y L), |t / s| <= L (1 + 2^-24),
// q = fl(t * fl(1/s)) and the IEEE quotient fl(t / s) each carry relative
// rounding errors of at most 2^-24 (two for q, one for the quotient), so
// they differ by less than 3.001 L 2^-24 < quant_margin(L).  Whenever q is
// at least that margin away from the nearest half-integer both round to the
// same integer (never beyond +-L), and rint(q) is the code.  Any value
// closer to a half-integer, a non-finite q, or a scale outside
// [2^-126, 2^125] (where 1/s could lose precision) sends the whole vector
// through the IEEE division.
template <int BITS>
__device__ __forceinline__ void quantize32(const float y[32], float s, uint32_t u[32])
{
    constexpr int L = (1 << (BITS - 1)) - 1;
    if (s == 0.f) {
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = (uint32_t)L;
        return;
    }
    bool slow = !(s > 2.350988701644575e-38f * 0.5f && s < 4.2535295865117308e37f);  // 2^-126 .. 2^125
    const float r = __frcp_rn(s);
    // |q| < 2^22: q + 1.5 2^23 lies in [2^23, 2^24), where the fp32 spacing is
    // 1, so the sum is rounded to the nearest integer n (ties to even, as
    // rintf), its bit pattern is that of 1.5 2^23 plus n, and subtracting
    // 1.5 2^23 again gives n exactly
    constexpr float kRound = 12582912.f;                 // 1.5 2^23 = 0x4B400000
    constexpr uint32_t kBias = 0x4B400000u - (uint32_t)L; // bits(kRound + n) - kBias = n + L
    const unsigned long long L2 = pk2((float)L, (float)L), r2 = pk2(r, r);
    const unsigned long long m2 = pk2(kRound, kRound);
    constexpr float kThr = 0.5f - quant_margin(L);          // exact in fp32
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        const unsigned long long t2 = mul2(pk2(y[i], y[i + 1]), L2);
        const unsigned long long q2 = mul2(t2, r2);
        const unsigned long long n2 = add2(q2, m2);          // kRound + rint(q)
        float d0, d1, n0, n1;
        up2(sub2(q2, sub2(n2, m2)), d0, d1);                  // q - rint(q), exact
        slow |= !(fabsf(d0) <= kThr) | !(fabsf(d1) <= kThr);
        up2(n2, n0, n1);
        u[i] = __float_as_uint(n0) - kBias;
        u[i + 1] = __float_as_uint(n1) - kBias;
    }
    if (slow) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            float c = roundf(__fdiv_rn(__fmul_rn(y[i], (float)L), s));
            c = fminf(fmaxf(c, -(float)L), (float)L);
            u[i] = (uint32_t)((int)c + L);
        }
    }
}

// fp8 codes of this thread's 32 values x (scale s = the vector's absmax):
// the E4M3 code nearest fl(fl(x 448) / s) (IEEE division), ties to the even
// mantissa, saturating at 448 (cvt .rn.satfinite); s == 0 gives codes 0.
__device__ __forceinline__ void quantize32_fp8(const float x[32], float s, uint32_t u[32])
{
    if (s == 0.f) {
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = 0u;
        return;
    }
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        const float y0 = __fdiv_rn(__fmul_rn(x[i], 448.f), s);
        const float y1 = __fdiv_rn(__fmul_rn(x[i + 1], 448.f), s);
        uint16_t pair;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(y1), "f"(y0));
        u[i] = pair & 0xFFu;             // the second operand (y0) lands in the low byte
        u[i + 1] = pair >> 8;
    }
}

// A token's slot continues the previous token's run: both valid, the next
// slot of the same page.
__device__ __forceinline__ bool continues(int64_t prev, int64_t cur, int page_size)
{
    return prev >= 0 && cur >= 0 && cur == prev + 1 && (cur & (page_size - 1)) != 0;
}

// First token index >= j that starts a run (or num_tokens); one warp.
__device__ __forceinline__ int64_t run_aligned(const int64_t* slots, int64_t j, int64_t num_tokens,
                                               int page_size, int lane)
{
    if (j <= 0) return 0;
    for (int64_t base = j; base < num_tokens; base += 32) {
        const int64_t t = base + lane;
        bool start = true;
        if (t < num_tokens) start = !continues(__ldg(slots + t - 1), __ldg(slots + t), page_size);
        const unsigned m = __ballot_sync(kFull, start);
        if (m) return min(num_tokens, base + __ffs(m) - 1);
    }
    return num_tokens;
}

// FP8: E4M3 codes with no rotation, in the 8-bit layout (BITS == 8).
template <int BITS, bool FP8 = false>
__global__ void __launch_bounds__(kQaThreads, 3)
k_quantize_append(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                  const int64_t* __restrict__ slots, int64_t num_tokens, int num_kv_heads,
                  int page_size, int lp, int num_pages, int block_bytes, int win, int hpc,
                  uint8_t* __restrict__ pool, uint32_t* err)
{
    constexpr int CB = kHeadDim * BITS / 8;            // K row bytes
    extern __shared__ __align__(16) uint8_t s_in[];    // [stage][chunk][thread][16 B] input ring
    __shared__ __align__(16) uint8_t s_v[2][kHeadDim * kVRow];   // [head & 1][dim][token ^ 8 (dim / 32)]
    __shared__ int s_page[kQaMaxWin], s_off[kQaMaxWin], s_run[kQaMaxWin];
    __shared__ int s_rs[kQaMaxWin], s_rlen[kQaMaxWin];  // runs: first window token, length
    __shared__ int s_ritem[kQaMaxWin + 1];              // runs: first V work item
    __shared__ int s_warp[8], s_nrun;
    __shared__ int64_t s_win[2];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head0 = blockIdx.y * hpc;                // heads [head0, head0 + hpc)
    const int P = page_size;

    // ---- the window, moved to run boundaries
    if (warp < 2) {
        const int64_t w = run_aligned(slots, ((int64_t)blockIdx.x + warp) * win, num_tokens, P,
                                      lane);
        if (lane == 0) s_win[warp] = w;
    }
    __syncthreads();
    const int64_t w0 = s_win[0];
    const int n = (int)(s_win[1] - w0);                // tokens of this window (<= 127)
    if (n <= 0) return;

    // ---- per token: page, offset, run starts and run ids
    int start = 0;
    if (tid < kQaMaxWin) {
        int pg = -1, off = 0;
        if (tid < n) {
            const int64_t sl = __ldg(slots + w0 + tid);
            if (sl >= 0) {
                const int64_t page = sl >> lp;
                if (page < num_pages) {
                    pg = (int)page;
                    off = (int)(sl & (P - 1));
                } else if (head0 == 0) {
                    report_error(err, TQ_ERR_DEVICE_CHECK, kErrSlotRange);
                }
            }
            start = pg >= 0 && (tid == 0 || !continues(__ldg(slots + w0 + tid - 1),
                                                        __ldg(slots + w0 + tid), P));
        }
        s_page[tid] = pg;
        s_off[tid] = off;
    }
    {
        // inclusive count of run starts over the window (tokens = threads 0..127)
        int x = start;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += s_warp[w];
        const int id = before + x - 1;                 // run of this token (if valid)
        if (tid < kQaMaxWin) s_run[tid] = s_page[tid] >= 0 ? id : -1;
        if (start) s_rs[id] = tid;
        if (tid == kQaThreads - 1) s_nrun = before + x;
        __syncthreads();
        if (tid < n && s_page[tid] >= 0) {
            const bool last = tid + 1 >= n || s_run[tid + 1] != id;
            if (last) s_rlen[id] = tid + 1 - s_rs[id];
        }
        __syncthreads();                               // run lengths are read by other threads
    }

    // ---- V: dim-major rows of every run.  A run that is a whole page in
    // order (its first window token a multiple of 8) writes the page's code
    // area in units of 16 bytes (12 bytes = 32 fields for 3-bit codes); any
    // other run writes, per dimension row, the words holding its fields.
    // The work items of all runs are spread over the CTA's threads.
    const int nrun = s_nrun;
    constexpr int kUnitFields = BITS == 3 ? 32 : 128 / BITS;        // fields per unit
    const int full_units = kHeadDim * P / kUnitFields;
    {
        int cnt = 0;
        if (tid < nrun) cnt = s_rlen[tid] == P ? full_units : kHeadDim;
        int x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += s_warp[w];
        if (tid < nrun) s_ritem[tid] = before + x - cnt;
        if (tid == kQaThreads - 1) s_ritem[kQaMaxWin] = before + x;     // total
        __syncthreads();
    }
    auto write_v_rows = [&](int head, const uint8_t* sv) {
    const int total = s_ritem[kQaMaxWin];
    for (int item = tid; item < total; item += kQaThreads) {
        int lo = 0, hi = nrun - 1;                       // the run: last s_ritem[r] <= item
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_ritem[mid] <= item) lo = mid;
            else hi = mid - 1;
        }
        const int r = lo, sub = item - s_ritem[r];
        const int rs = s_rs[r], len = s_rlen[r];
        const int page = s_page[rs], o1 = s_off[rs];
        uint32_t* code = reinterpret_cast<uint32_t*>(
            pool + ((int64_t)(page * num_kv_heads + head) * 2 + 1) * block_bytes);
        if (len == P) {
            // unit `sub`: fields kUnitFields * sub ... in code-area order; a
            // group of 8 fields is one dimension row's 8 consecutive tokens,
            // read as the aligned 8-byte group(s) holding them
            const int f0 = kUnitFields * sub;
            auto group8 = [&](int f, uint32_t& lo4, uint32_t& hi4) {
                const int d = f / P, off = f - d * P;
                const uint8_t* row = sv + d * kVRow;
                const int x8 = 8 * (d >> 5), c = rs + off, a = c & ~7, o = c & 7;
                const uint2 A = *reinterpret_cast<const uint2*>(row + (a ^ x8));
                if (o == 0) {
                    lo4 = A.x;
                    hi4 = A.y;
                    return;
                }
                const uint2 B = *reinterpret_cast<const uint2*>(row + ((a + 8) ^ x8));
                const uint32_t sel = 0x3210u + 0x1111u * (uint32_t)(o & 3);
                lo4 = o < 4 ? __byte_perm(A.x, A.y, sel) : __byte_perm(A.y, B.x, sel);
                hi4 = o < 4 ? __byte_perm(A.y, B.x, sel) : __byte_perm(B.x, B.y, sel);
            };
            if constexpr (BITS == 3) {
                uint32_t g[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t a, b;
                    group8(f0 + 8 * j, a, b);
                    auto pack3 = [](uint32_t x) {   // 4 bytes < 8 -> 12 bits
                        return (x & 0x7u) | ((x >> 5) & 0x38u) | ((x >> 10) & 0x1C0u) |
                               ((x >> 15) & 0xE00u);
                    };
                    g[j] = pack3(a) | (pack3(b) << 12);
                }
                uint32_t* dst = code + 3 * sub;
                dst[0] = g[0] | (g[1] << 24);
                dst[1] = (g[1] >> 8) | (g[2] << 16);
                dst[2] = (g[2] >> 16) | (g[3] << 8);
            } else {
                uint32_t wd[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int f = f0 + e * (32 / BITS);          // first field of word e
                    if constexpr (BITS == 8) {
                        if ((e & 1) == 0) {                      // words e, e + 1: 8 fields
                            uint32_t a, b;
                            group8(f, a, b);
                            wd[e] = a;
                            wd[e + 1] = b;
                        }
                    } else if constexpr (BITS == 4) {
                        uint32_t a, b;
                        group8(f, a, b);
                        a |= a >> 4;
                        b |= b >> 4;
                        wd[e] = __byte_perm(a, b, 0x6420);
                    } else {  // 2 bits: 16 fields = two groups of 8
                        uint32_t in[4];
                        group8(f, in[0], in[1]);
                        group8(f + 8, in[2], in[3]);
                        uint32_t o = 0;
#pragma unroll
                        for (int gq = 0; gq < 4; ++gq) {
                            uint32_t y = in[gq] | (in[gq] >> 6);      // bytes 0, 2: 4 bits each
                            y = (y & 0xFFu) | ((y >> 12) & 0xF0u);   // 8 bits: 4 fields
                            o |= y << (8 * gq);
                        }
                        wd[e] = o;
                    }
                }
                reinterpret_cast<uint4*>(code)[sub] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            }
        } else {
            // dimension row `sub`: fields [o1, o1 + len) of the row, in bit
            // order; a word entirely ours is stored, a shared one merged
            const int d = sub;
            const uint32_t fm = (1u << BITS) - 1u;
            int64_t cw = ((int64_t)d * P * BITS + (int64_t)o1 * BITS) >> 5;
            uint32_t val = 0, msk = 0;
            auto flush = [&]() {
                if (msk == 0xFFFFFFFFu) {
                    code[cw] = val;
                } else if (msk) {
                    atomicAnd(code + cw, ~msk);
                    atomicOr(code + cw, val);
                }
            };
            for (int f = 0; f < len; ++f) {
                const int64_t fb = (int64_t)d * P * BITS + (int64_t)(o1 + f) * BITS;
                const int64_t w = fb >> 5;
                const int sh = (int)(fb & 31);
                if (w != cw) {
                    flush();
                    cw = w;
                    val = msk = 0;
                }
                const uint32_t uu = sv[d * kVRow + ((rs + f) ^ (8 * (d >> 5)))];
                val |= uu << sh;
                msk |= fm << sh;
                if (sh + BITS > 32) {                 // a 3-bit field across two words
                    flush();
                    cw = w + 1;
                    val = uu >> (32 - sh);
                    msk = fm >> (32 - sh);
                }
            }
            flush();
        }
    }
    };
    // ---- quantise: passes of 32 tokens of one head, warps 0-3 K, warps 4-7 V;
    // each thread fetches its 64 input bytes of the next pass by cp.async
    // into its own slot of a 2-stage ring while it computes this one
    const int which = warp >> 2;
    const int q = lane & 3;
    const int vi = (warp & 3) * 8 + (lane >> 2);        // vector of the pass (token in chunk)
    const int nchunk = (n + kQaPass - 1) / kQaPass;
    const int npass = hpc * nchunk;
    auto issue = [&](int pidx) {
        if (pidx < npass) {
            const int hh = pidx / nchunk, tk = (pidx - hh * nchunk) * kQaPass + vi;
            if (tk < n) {
                const uint16_t* src = (which ? v : k) +
                                      ((w0 + tk) * num_kv_heads + head0 + hh) * kHeadDim + 32 * q;
                // ring slot [stage][chunk][thread]: a warp's 16-byte chunks are contiguous
                uint8_t* dst = s_in + ((pidx % kQaStages) * 4 * kQaThreads + tid) * 16;
#pragma unroll
                for (int c = 0; c < 4; ++c) cp_async16(dst + c * kQaThreads * 16, src + 8 * c);
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int p = 0; p < kQaStages - 1; ++p) issue(p);
    for (int pidx = 0; pidx < npass; ++pidx) {
        issue(pidx + kQaStages - 1);
        cp_async_wait<kQaStages - 1>();                  // this pass's bytes have landed
        const int hh = pidx / nchunk, chunk = pidx - hh * nchunk;
        const int head = head0 + hh;
        const int tk = chunk * kQaPass + vi;                                  // window token
        const bool live = tk < n && s_page[tk] >= 0;
        float x[32];
        if (tk < n) {
            const uint4* src = reinterpret_cast<const uint4*>(s_in) +
                               (pidx % kQaStages) * 4 * kQaThreads + tid;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 raw = src[c * kQaThreads];
                const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * c + 2 * e] = __uint_as_float(wd[e] << 16);
                    x[8 * c + 2 * e + 1] = __uint_as_float(wd[e] & 0xffff0000u);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = 0.f;
        }
        if constexpr (!FP8) {
            fwht32_in_thread(x);
            fwht32_across(x, q);
            const float c = __uint_as_float(0x3DB504F3u);   // fp32(1 / sqrt(128))
            const unsigned long long c2 = pk2(c, c);
#pragma unroll
            for (int i = 0; i < 32; i += 2) up2(mul2(pk2(x[i], x[i + 1]), c2), x[i], x[i + 1]);
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 2) amax = fmaxf(amax, fmaxf(fabsf(x[i]), fabsf(x[i + 1])));
        amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
        uint32_t u[32];
        if constexpr (FP8) quantize32_fp8(x, amax, u);
        else quantize32<BITS>(x, amax, u);
        if (live) {
            const int page = s_page[tk], off = s_off[tk];
            uint8_t* blk = pool + ((int64_t)(page * num_kv_heads + head) * 2 + which) * block_bytes;
            if (q == 0) *reinterpret_cast<float*>(blk + P * CB + 4 * off) = amax;
            if (which == 0) {
                // K: this thread's piece of token row `off`
                uint8_t* row = blk + off * CB;
                const int sw = k_swizzle<BITS>(off);
                if constexpr (BITS == 4) {
                    uint32_t wd[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t acc = 0;
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc |= u[8 * j + i] << (4 * i);
                        wd[j] = acc;
                    }
                    *reinterpret_cast<uint4*>(row + 16 * (q ^ sw)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                } else if constexpr (BITS == 8) {
                    uint32_t wd[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        wd[j] = u[4 * j] | (u[4 * j + 1] << 8) | (u[4 * j + 2] << 16) | (u[4 * j + 3] << 24);
                    *reinterpret_cast<uint4*>(row + 16 * ((2 * q) ^ sw)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                    *reinterpret_cast<uint4*>(row + 16 * ((2 * q + 1) ^ sw)) = make_uint4(wd[4], wd[5], wd[6], wd[7]);
                } else if constexpr (BITS == 2) {
                    uint32_t wd[2];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        uint32_t acc = 0;
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc |= u[16 * j + i] << (2 * i);
                        wd[j] = acc;
                    }
                    *reinterpret_cast<uint2*>(row + 16 * ((q >> 1) ^ sw) + 8 * (q & 1)) = make_uint2(wd[0], wd[1]);
                } else {  // 3 bits: 12 bytes at 12 q, rows stored in order
                    uint32_t wd[3] = {0u, 0u, 0u};
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int pos = 3 * i, wi = pos >> 5, sh = pos & 31;
                        wd[wi] |= u[i] << sh;
                        if (sh > 29) wd[wi + 1] |= u[i] >> (32 - sh);
                    }
                    uint32_t* dst = reinterpret_cast<uint32_t*>(row + 12 * q);
                    dst[0] = wd[0];
                    dst[1] = wd[1];
                    dst[2] = wd[2];
                }
            } else {
                // V: stage u dimension-major, column tk ^ 8q
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    s_v[hh & 1][(32 * q + i) * kVRow + (tk ^ (8 * q))] = (uint8_t)u[i];
            }
        }
        if (chunk == nchunk - 1) {
            // head `head` is staged, and every thread is done writing the
            // previous head from the other buffer, which the next head fills
            __syncthreads();
            write_v_rows(head, s_v[hh & 1]);
        }
    }
    cp_async_wait<0>();
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

template <int BITS, bool FP8 = false>
cudaError_t launch_qa(const uint16_t* k, const uint16_t* v, const int64_t* slots, int num_tokens,
                      const tq_cache& c, int lp, int block_bytes, int win, int hpc,
                      uint8_t* pool, int dev, cudaStream_t stream)
{
    static unsigned configured = 0;                // one bit per device ordinal < 32
    if (dev >= 32 || !(configured & (1u << dev))) {
        cudaError_t e = cudaFuncSetAttribute(k_quantize_append<BITS, FP8>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kQaInBytes);
        if (e != cudaSuccess) return e;
        if (dev < 32) configured |= 1u << dev;
    }
    const dim3 grid((unsigned)((num_tokens + win - 1) / win), (unsigned)(c.num_kv_heads / hpc));
    k_quantize_append<BITS, FP8><<<grid, kQaThreads, kQaInBytes, stream>>>(
        k, v, slots, num_tokens, c.num_kv_heads, c.page_size, lp, c.num_pages, block_bytes, win,
        hpc, pool, c.dev_error);
    return cudaGetLastError();
}

cudaError_t launch_quantize_append(const void* k, const void* v, const int64_t* slots,
                                   int num_tokens, int bits, const tq_cache& c,
                                   int64_t block_bytes, cudaStream_t stream)
{
    // large calls: windows of 64 tokens with every kv head in one CTA (the
    // window scans done once); small ones (per-step appends): windows of 8
    // tokens and one head per CTA, for more CTAs with less work each
    static int nsm_of[32] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int nsm = dev < 32 ? nsm_of[dev] : 0;
    if (nsm == 0) {
        e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        if (dev < 32) nsm_of[dev] = nsm;
    }
    const bool large = ((int64_t)num_tokens + kQaWin - 1) / kQaWin >= 2 * nsm;
    const int win = large ? kQaWin : 8;
    const int hpc = large ? c.num_kv_heads : 1;
    const auto* kk = static_cast<const uint16_t*>(k);
    const auto* vv = static_cast<const uint16_t*>(v);
    auto* pool = static_cast<uint8_t*>(c.pages);
    const int lp = c.page_size == 16 ? 4 : (c.page_size == 32 ? 5 : 6);
    const int bb = (int)block_bytes;
    switch (bits) {
    case 2: return launch_qa<2>(kk, vv, slots, num_tokens, c, lp, bb, win, hpc, pool, dev, stream);
    case 3: return launch_qa<3>(kk, vv, slots, num_tokens, c, lp, bb, win, hpc, pool, dev, stream);
    case 4: return launch_qa<4>(kk, vv, slots, num_tokens, c, lp, bb, win, hpc, pool, dev, stream);
    case 8: return launch_qa<8>(kk, vv, slots, num_tokens, c, lp, bb, win, hpc, pool, dev, stream);
    case TQ_FP8:
        return launch_qa<8, true>(kk, vv, slots, num_tokens, c, lp, bb, win, hpc, pool, dev, stream);
    default: return cudaErrorInvalidValue;
    }
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
