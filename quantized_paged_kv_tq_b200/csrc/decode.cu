// Paged decode / speculative-verify attention over the bf16 cache: the
// uncompressed reference point beside the TurboQuant decode (decode_tc.cu),
// and the split-size / workspace bookkeeping both decodes share.
//
// "infero", section "Continuous batching": a running batch shares the GPU
// over a paged KV cache.
//
// Work decomposition (split-KV):
//   grid = (max splits, kv heads x row groups, batch), 4 warps per CTA.
//   A CTA owns one (sequence, kv head, row group, split); a split is a fixed
//   run of 2048 tokens (1024 for 64-token pages), so a sequence's result
//   never depends on the rest of the batch.  All G = q_len * GQA query rows
//   of the kv head (up to 8 per row group) share every byte read.
//   Each warp streams its own 16-token tiles (tile w, w+4, ...) through a
//   private ring of shared-memory stages filled by 1-D bulk async copies
//   (cp.async.bulk + mbarrier) of the K and V rows.
//
// Per tile (16 tokens):
//   QK^T  mma.sync m16n8k16 with bf16 K rows as A and the query (scaled to
//         log2 units, power-of-two prescale) split into bf16 hi + lo
//         columns as B; fp32 accumulate.
//   softmax online, with a lazy rescale: the running max only moves when a
//         tile exceeds it by 2^8; causal limit j <= seq_len - q_len + t.
//   PV    mma.sync with A = V rows (dims on M, tokens on K) and B = P split
//         into bf16 hi + lo, transposed in registers by movmatrix.
// Epilogue: the 4 warps merge in shared memory; a sequence with one split
// finishes directly, otherwise the CTA stores (m, l, O) partials and the last
// CTA of the (sequence, kv head, row group), found with an atomic ticket,
// merges all splits and writes fp32 output.
#include <cstdint>
#include <math_constants.h>

#include "tq_device.cuh"

namespace tq {

namespace {

// Tuning constants (compile-time; the defaults are the measured choice).
#ifndef TQ_SPLIT_TOKENS
#define TQ_SPLIT_TOKENS 2048      // tokens per split-KV part (pages of 16/32), <= 2048
#endif
#ifndef TQ_SPLIT_TOKENS_P64
#define TQ_SPLIT_TOKENS_P64 1024  // 64-token pages: >= 128 parts for a 131072-token context
#endif
#ifndef TQ_STAGE_BUDGET
#define TQ_STAGE_BUDGET 6528      // target bytes of one warp's staging ring
#endif
#ifndef TQ_MAX_STAGES
#define TQ_MAX_STAGES 3
#endif
static_assert(TQ_SPLIT_TOKENS % 64 == 0 && TQ_SPLIT_TOKENS <= 2048 &&
                  TQ_SPLIT_TOKENS_P64 % 64 == 0 && TQ_SPLIT_TOKENS_P64 <= 2048,
              "a warp holds the page ids of its tiles in one register per lane");

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxStages = TQ_MAX_STAGES;
// shared memory header: q rows [8][128] fp32, row factors, flags, mbarriers
constexpr int kBarOff = 4224;
constexpr int kRingOff = (kBarOff + 8 * 4 * kMaxStages + 127) / 128 * 128;
constexpr int kRowsPerCta = 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazyThreshold = 8.f;       // log2 units
constexpr uint32_t kWaitSpins = 1u << 24;   // bounded mbarrier polls

struct DecodeArgs {
    const uint16_t* q;
    const uint8_t* kv;         // pool[page][kv head][K block, V block]
    const int32_t* page_table;
    const int32_t* seq_lens;
    float* out;
    float* ws_o;
    float2* ws_ml;
    uint32_t* ws_cnt;
    uint32_t* err;
    int64_t block_bytes;
    int max_pages;
    int num_pages;
    int num_kv_heads;
    int num_q_heads;
    int group;
    int q_len;
    int G;          // query rows per kv head
    int R;          // row groups of <= 8 rows
    int page_size;
    int split_tokens;
    int max_splits;
    int max_seq_len;
    int stages;
};

// Staging of the bf16 cache: 16 token rows of d bf16 values for K, then V.
template <int BITS>
struct Fmt {
    static_assert(BITS == 16, "the mma.sync kernel serves the bf16 cache");
    static constexpr int CB = 2 * kHeadDim;            // row bytes
    static constexpr int kTileCodes = 16 * CB;
    static constexpr int kVOff = kTileCodes;
    static constexpr int kStageBytes = 2 * kVOff;
};

// QK^T tile row r (0..15) holds tile token perm(r); chosen so that the
// transposed probabilities land on the PV B-fragment (tokens t, t+4, t+8,
// t+12 for lane group t) and shared-memory reads spread over banks.
__device__ __forceinline__ int perm(int r)
{
    return (r & 8) | ((r & 1) << 2) | ((r >> 1) & 3);
}

// Head dimension held by fragment element (chunk c, k = 2t + e + 8f) of the
// QK^T operands; it follows the order the unpacker produces values in.
template <int BITS>
__device__ __forceinline__ int qk_dim(int t, int c, int f, int e)
{
    return 32 * t + 8 * (c >> 1) + 4 * (c & 1) + 2 * f + e;
}

// ----------------------------------------------------------- K rows
// ka[c][f]: bf16x2 A-fragment element pair for chunk c, half f, of one token
// row (dims 32t .. 32t + 31, adjacent pairs as stored); `row` points at that
// token's row in the stage.
template <int BITS>
__device__ __forceinline__ void unpack_k(const uint8_t* row, int t, uint32_t ka[8][2])
{
#pragma unroll
    for (int w4 = 0; w4 < 4; ++w4) {
        const uint4 x = *reinterpret_cast<const uint4*>(row + 64 * t + 16 * w4);
        ka[2 * w4][0] = x.x;
        ka[2 * w4][1] = x.y;
        ka[2 * w4 + 1][0] = x.z;
        ka[2 * w4 + 1][1] = x.w;
    }
}

// ----------------------------------------------------------- V rows
// va[mt][i]: A-fragment of V^T for m-tile mt (rows = dims 16g + 2mt and
// 16g + 2mt + 1), k = tokens {t, t+4} (i = 0, 1) and {t+8, t+12} (i = 2, 3).
template <int BITS>
__device__ __forceinline__ void unpack_v(const uint8_t* codes, int g, int t, uint32_t va[8][4])
{
    constexpr int CB = Fmt<BITS>::CB;
    const uint8_t* r0 = codes + (t + 0) * CB;
    const uint8_t* r1 = codes + (t + 4) * CB;
    const uint8_t* r2 = codes + (t + 8) * CB;
    const uint8_t* r3 = codes + (t + 12) * CB;
    uint4 X[4][2];
    const uint8_t* rows[4] = {r0, r1, r2, r3};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        X[i][0] = *reinterpret_cast<const uint4*>(rows[i] + 32 * g);
        X[i][1] = *reinterpret_cast<const uint4*>(rows[i] + 32 * g + 16);
    }
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        const uint32_t xa[8] = {X[2 * p][0].x, X[2 * p][0].y, X[2 * p][0].z, X[2 * p][0].w,
                                X[2 * p][1].x, X[2 * p][1].y, X[2 * p][1].z, X[2 * p][1].w};
        const uint32_t ya[8] = {X[2 * p + 1][0].x, X[2 * p + 1][0].y, X[2 * p + 1][0].z,
                                X[2 * p + 1][0].w, X[2 * p + 1][1].x, X[2 * p + 1][1].y,
                                X[2 * p + 1][1].z, X[2 * p + 1][1].w};
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            va[mt][2 * p] = prmt(xa[mt], ya[mt], 0x5410u);
            va[mt][2 * p + 1] = prmt(xa[mt], ya[mt], 0x7632u);
        }
    }
}

template <int BITS>
__device__ __forceinline__ void issue_tile(uint8_t* dst, uint64_t* bar, const DecodeArgs& a,
                                           int page, int kvh, int sub, bool one_block)
{
    using F = Fmt<BITS>;
    const int64_t blk = ((int64_t)page * a.num_kv_heads + kvh) * 2 * a.block_bytes;
    const uint8_t* kb = a.kv + blk;
    const uint8_t* vb = kb + a.block_bytes;
    mbar_arrive_expect_tx(bar, F::kStageBytes);
    if (one_block) {
        // a 16-token page is exactly one tile
        bulk_g2s(dst, kb, F::kVOff, bar);
        bulk_g2s(dst + F::kVOff, vb, F::kVOff, bar);
        return;
    }
    bulk_g2s(dst, kb + sub * F::kTileCodes, F::kTileCodes, bar);
    bulk_g2s(dst + F::kVOff, vb + sub * F::kTileCodes, F::kTileCodes, bar);
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kThreads)
k_decode(const DecodeArgs a)
{
    using F = Fmt<BITS>;
    extern __shared__ __align__(128) uint8_t smem[];
    float* sQ = reinterpret_cast<float*>(smem);                      // [8][128]
    float* sRowFac = sQ + kRowsPerCta * kHeadDim;                    // [8]
    int* sFlag = reinterpret_cast<int*>(sRowFac + 16);               // [4]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);    // [4][kMaxStages]
    uint8_t* ring = smem + kRingOff;

    const int split = blockIdx.x;
    const int b = blockIdx.z;
    const int kvh = blockIdx.y / a.R;
    const int rg = blockIdx.y - kvh * a.R;
    const int seq_len = a.seq_lens[b];
    if (seq_len < a.q_len || seq_len > a.max_seq_len) {
        if (split == 0 && blockIdx.y == 0 && threadIdx.x == 0)
            report_error(a.err, TQ_ERR_DEVICE_CHECK, kErrSeqLen);
        return;
    }
    const int nsplit = (seq_len + a.split_tokens - 1) / a.split_tokens;
    if (split >= nsplit) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tok_begin = split * a.split_tokens;
    const int tok_end = min(seq_len, tok_begin + a.split_tokens);
    const int ntiles = (tok_end - tok_begin + 15) >> 4;
    const int my_tiles = ntiles > warp ? (ntiles - warp + kWarps - 1) / kWarps : 0;
    const int stages = a.stages;
    uint64_t* mybar = bars + warp * kMaxStages;
    uint8_t* myring = ring + warp * stages * F::kStageBytes;

    // physical page of each of my tiles: lane j holds tile j
    int pid = 0, psub = 0;
    if (lane < my_tiles) {
        const int tok = tok_begin + 16 * (warp + kWarps * lane);
        pid = __ldg(a.page_table + (int64_t)b * a.max_pages + tok / a.page_size);
        psub = (tok % a.page_size) >> 4;
        if (pid < 0 || pid >= a.num_pages) {
            report_error(a.err, TQ_ERR_DEVICE_CHECK, kErrPageRange);
            pid = 0;
        }
    }
    if (lane == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&mybar[s], 1);
        fence_barrier_init();
    }
    if (threadIdx.x == 0) sFlag[0] = 0;
    __syncwarp();
    const int first = min(stages, my_tiles);
    for (int i = 0; i < first; ++i) {
        const int p = __shfl_sync(kFull, pid, i);
        const int sb = __shfl_sync(kFull, psub, i);
        if (lane == 0)
            issue_tile<BITS>(myring + i * F::kStageBytes, &mybar[i], a, p, kvh, sb,
                             a.page_size == 16);
    }

    // ---- rotated, scaled query rows of this row group (while tiles load)
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int rr = warp + 4 * k;
        const int r = rg * kRowsPerCta + rr;
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (r < a.G) {
            const int tq = r / a.group;
            const int h = kvh * a.group + (r - tq * a.group);
            const uint2 raw = __ldg(reinterpret_cast<const uint2*>(
                a.q + (((int64_t)b * a.q_len + tq) * a.num_q_heads + h) * kHeadDim) + lane);
            x[0] = bf16_bits_to_float(raw.x & 0xffffu);
            x[1] = bf16_bits_to_float(raw.x >> 16);
            x[2] = bf16_bits_to_float(raw.y & 0xffffu);
            x[3] = bf16_bits_to_float(raw.y >> 16);
        }
        const float fac = kLog2e * 0.08838834764831845f;  // 1 / sqrt(128)
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[e] *= fac;
            amax = fmaxf(amax, fabsf(x[e]));
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, m));
        // power-of-two prescale: largest |q'| in [2^12, 2^13) keeps hi and lo
        // f16 parts normal; the inverse factor is applied to the scores
        const int ex = amax > 0.f ? max(-100, min(100, ilogbf(amax))) : 0;
        const float pre = pow2i(12 - ex);
#pragma unroll
        for (int e = 0; e < 4; ++e) sQ[rr * kHeadDim + 4 * lane + e] = x[e] * pre;
        if (lane == 0) sRowFac[rr] = pow2i(ex - 12);
    }
    __syncthreads();

    // B fragments of the query: column n = g holds row 4nt + (g & 3), hi
    // part for g < 4, lo part for g >= 4
    uint32_t qf[NT][8][2];
    float rowfac[NT][2];
    int lim[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const float* qrow = sQ + (4 * nt + (g & 3)) * kHeadDim;
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
            for (int f = 0; f < 2; ++f) {
                const float v0 = qrow[qk_dim<BITS>(t, c, f, 0)];
                const float v1 = qrow[qk_dim<BITS>(t, c, f, 1)];
                const float h0 = __bfloat162float(__float2bfloat16_rn(v0));
                const float h1 = __bfloat162float(__float2bfloat16_rn(v1));
                qf[nt][c][f] = g < 4 ? pack_bf162(v0, v1) : pack_bf162(v0 - h0, v1 - h1);
            }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int rl = 4 * nt + 2 * (t & 1) + e;
            const int r = rg * kRowsPerCta + rl;
            rowfac[nt][e] = sRowFac[rl];
            lim[nt][e] = r < a.G ? seq_len - a.q_len + r / a.group : -1;
        }
    }

    float o[NT][8][4];
    float m_run[NT][2], l_run[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[nt][mt][i] = 0.f;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            m_run[nt][e] = -CUDART_INF_F;
            l_run[nt][e] = 0.f;
        }
    }
    const int ra = perm(g), rb = perm(g + 8);
    // a tile is fully visible when its last token is within the causal limit
    // of the first (most restricted) row of this row group
    const int lim_min = seq_len - a.q_len + (rg * kRowsPerCta) / a.group;
    const bool one_block = a.page_size == 16;

    int failed_at = -1;
    int slot = 0;
    uint32_t phase = 0;
    int tok0 = tok_begin + 16 * warp;
    for (int i = 0; i < my_tiles; ++i, tok0 += 16 * kWarps) {
        if (!mbar_wait_bounded(&mybar[slot], phase, kWaitSpins)) {
            if (lane == 0) report_error(a.err, TQ_ERR_TIMEOUT, kErrWaitTile);
            failed_at = i;
            break;
        }
        const uint8_t* st = myring + slot * F::kStageBytes;

        // ---------------- S = K q'  (two independent accumulation chains)
        float s[NT][4];
        {
            float s2[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int k = 0; k < 4; ++k) s[nt][k] = s2[nt][k] = 0.f;
            uint32_t ka[8][2], kb[8][2];
            unpack_k<BITS>(st + ra * F::CB, t, ka);
            unpack_k<BITS>(st + rb * F::CB, t, kb);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t afr[4] = {ka[c][0], kb[c][0], ka[c][1], kb[c][1]};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float* acc = c < 4 ? s[nt] : s2[nt];
                    mma_bf16(acc, afr, qf[nt][c][0], qf[nt][c][1]);
                }
            }
            // hi + lo columns (lanes t and t ^ 2)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    s[nt][k] += s2[nt][k];
                    s[nt][k] += __shfl_xor_sync(kFull, s[nt][k], 2);
                }
        }
        // 1 for a token of the sequence, 0 for a slot past its end
        float ks0 = 1.f, ks1 = 1.f, vs0 = 1.f, vs1 = 1.f;
        const bool full = tok0 + 15 <= lim_min;     // warp-uniform
        const int ja = tok0 + ra, jb = tok0 + rb;
        if (!full) {
            // slots past the sequence end were never written: keep them out
            // of every product
            if (ja >= seq_len) { ks0 = 0.f; vs0 = 0.f; }
            if (jb >= seq_len) { ks1 = 0.f; vs1 = 0.f; }
        }
        // scores in log2 units; masked entries -inf (only in partial tiles)
        float sc[NT][4];
        bool need = false;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float x0 = s[nt][e] * (ks0 * rowfac[nt][e]);
                float x1 = s[nt][2 + e] * (ks1 * rowfac[nt][e]);
                if (!full) {
                    x0 = ja <= lim[nt][e] ? x0 : -CUDART_INF_F;
                    x1 = jb <= lim[nt][e] ? x1 : -CUDART_INF_F;
                }
                sc[nt][e] = x0;
                sc[nt][2 + e] = x1;
                need |= fmaxf(x0, x1) > m_run[nt][e] + kLazyThreshold;
            }
        if (__any_sync(kFull, need)) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = fmaxf(sc[nt][e], sc[nt][2 + e]);
                    v = fmaxf(v, __shfl_xor_sync(kFull, v, 4));
                    v = fmaxf(v, __shfl_xor_sync(kFull, v, 8));
                    v = fmaxf(v, __shfl_xor_sync(kFull, v, 16));
                    const float mn = fmaxf(m_run[nt][e], v);
                    const float alpha = mn == -CUDART_INF_F ? 1.f : fast_exp2(m_run[nt][e] - mn);
                    m_run[nt][e] = mn;
                    l_run[nt][e] *= alpha;
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        o[nt][mt][e] *= alpha;
                        o[nt][mt][2 + e] *= alpha;
                    }
                }
        }
        // P, split into hi (lanes t < 2) and lo (t >= 2) bf16 halves,
        // transposed onto the PV B fragment
        const float vn0 = vs0, vn1 = vs1;
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float p0 = fast_exp2(sc[nt][e] - m_run[nt][e]);
                float p1 = fast_exp2(sc[nt][2 + e] - m_run[nt][e]);
                if (!full) {
                    // -inf - -inf would be NaN: masked entries are exactly 0
                    p0 = sc[nt][e] == -CUDART_INF_F ? 0.f : p0;
                    p1 = sc[nt][2 + e] == -CUDART_INF_F ? 0.f : p1;
                }
                l_run[nt][e] += p0 + p1;
                pv[e] = p0 * vn0;
                pv[2 + e] = p1 * vn1;
                if (!full) {
                    // a masked entry stays exactly 0
                    pv[e] = p0 > 0.f ? pv[e] : 0.f;
                    pv[2 + e] = p1 > 0.f ? pv[2 + e] : 0.f;
                }
            }
            pb[nt][0] = movmatrix_trans(split_hi_lo<false>(pv[0], pv[1], t < 2));
            pb[nt][1] = movmatrix_trans(split_hi_lo<false>(pv[2], pv[3], t < 2));
        }

        // ---------------- O^T += V^T P'
        {
            uint32_t va[8][4];
            unpack_v<BITS>(st + F::kVOff, g, t, va);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma_bf16(o[nt][mt], va[mt], pb[nt][0], pb[nt][1]);
                }
        }

        __syncwarp();
        if (i + stages < my_tiles) {
            const int p = __shfl_sync(kFull, pid, i + stages);
            const int sb = __shfl_sync(kFull, psub, i + stages);
            if (lane == 0)
                issue_tile<BITS>(myring + slot * F::kStageBytes, &mybar[slot], a, p, kvh, sb,
                                 one_block);
        }
        if (++slot == stages) {
            slot = 0;
            phase ^= 1u;
        }
    }

    if (failed_at >= 0) {
        // drain this warp's copies still in flight (bounded), then give up
        const int last = min(my_tiles, failed_at + stages);
        for (int j = failed_at + 1; j < last; ++j)
            (void)mbar_wait_bounded(&mybar[j % stages], (uint32_t)((j / stages) & 1), kWaitSpins);
        if (lane == 0) atomicExch(&sFlag[0], 1);
    }

    // ---- warp partials -> shared memory (the ring is free now)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float l = l_run[nt][e];
            l += __shfl_xor_sync(kFull, l, 4);
            l += __shfl_xor_sync(kFull, l, 8);
            l += __shfl_xor_sync(kFull, l, 16);
            l_run[nt][e] = l;
        }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                o[nt][mt][i] = o[nt][mt][i] + __shfl_xor_sync(kFull, o[nt][mt][i], 2);

    __syncthreads();  // every warp is done with its ring
    float* sO = reinterpret_cast<float*>(ring);                          // [4][8][128]
    float* sM = sO + kWarps * kRowsPerCta * kHeadDim;                    // [4][8]
    float* sL = sM + kWarps * kRowsPerCta;                               // [4][8]
    if (t < 2) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int rl = 4 * nt + 2 * t + e;
                float* dst = sO + (warp * kRowsPerCta + rl) * kHeadDim + 16 * g;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    dst[2 * mt] = o[nt][mt][e];
                    dst[2 * mt + 1] = o[nt][mt][2 + e];
                }
                if (g == 0) {
                    sM[warp * kRowsPerCta + rl] = m_run[nt][e];
                    sL[warp * kRowsPerCta + rl] = l_run[nt][e];
                }
            }
    }
    __syncthreads();
    // A CTA that gave up on a bounded wait (sFlag[0], CTA-uniform here) reads
    // none of its partials; in a multi-split sequence it still records an
    // empty partial and takes its ticket, so the counter wraps back to zero.
    const bool valid = sFlag[0] == 0;
    if (!valid && nsplit == 1) return;

    // ---- merge the 4 warps; warp w takes rows w and w + 4
    const int nrows = min(kRowsPerCta, min(4 * NT, a.G - rg * kRowsPerCta));
    const int64_t unit = ((int64_t)b * gridDim.y + blockIdx.y);        // (seq, kvh, rg)
    const int64_t part = unit * a.max_splits + split;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int rr = warp + 4 * k;
        if (rr >= nrows) continue;
        if (!valid) {
            if (lane == 0) a.ws_ml[part * kRowsPerCta + rr] = make_float2(-CUDART_INF_F, 0.f);
            continue;
        }
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sM[w * kRowsPerCta + rr]);
        float Lsum = 0.f;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float mw = sM[w * kRowsPerCta + rr];
            const float sc = mw == -CUDART_INF_F ? 0.f : exp2f(mw - M);
            Lsum += sc * sL[w * kRowsPerCta + rr];
            const float4 v = *reinterpret_cast<const float4*>(
                sO + (w * kRowsPerCta + rr) * kHeadDim + 4 * lane);
            acc[0] += sc * v.x;
            acc[1] += sc * v.y;
            acc[2] += sc * v.z;
            acc[3] += sc * v.w;
        }
        const int r = rg * kRowsPerCta + rr;
        const int tq = r / a.group;
        const int h = kvh * a.group + (r - tq * a.group);
        if (nsplit == 1) {
            const float inv = 1.f / Lsum;
            float x[4] = {acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv};
            *reinterpret_cast<float4*>(a.out + (((int64_t)b * a.q_len + tq) * a.num_q_heads + h) *
                                                   kHeadDim + 4 * lane) =
                make_float4(x[0], x[1], x[2], x[3]);
        } else {
            *reinterpret_cast<float4*>(a.ws_o + (part * kRowsPerCta + rr) * kHeadDim + 4 * lane) =
                make_float4(acc[0], acc[1], acc[2], acc[3]);
            if (lane == 0) a.ws_ml[part * kRowsPerCta + rr] = make_float2(M, Lsum);
        }
    }
    if (nsplit == 1) return;

    // ---- last CTA of this (seq, kv head, row group) merges every split
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned old = atomicInc(a.ws_cnt + unit, (unsigned)(nsplit - 1));
        sFlag[1] = old == (unsigned)(nsplit - 1);
    }
    __syncthreads();
    if (!sFlag[1]) return;
    __threadfence();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int rr = warp + 4 * k;
        if (rr >= nrows) continue;
        const int64_t base = unit * a.max_splits;
        float M = -CUDART_INF_F;
        for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, __ldcg(a.ws_ml + (base + sp) * kRowsPerCta + rr).x);
        float Lsum = 0.f;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int sp = 0; sp < nsplit; ++sp) {
            const float2 ml = __ldcg(a.ws_ml + (base + sp) * kRowsPerCta + rr);
            if (ml.x == -CUDART_INF_F) continue;       // empty split: no keys, no O written
            const float sc = exp2f(ml.x - M);
            Lsum += sc * ml.y;
            const float4 v = __ldcg(reinterpret_cast<const float4*>(
                a.ws_o + ((base + sp) * kRowsPerCta + rr) * kHeadDim) + lane);
            acc[0] += sc * v.x;
            acc[1] += sc * v.y;
            acc[2] += sc * v.z;
            acc[3] += sc * v.w;
        }
        const float inv = 1.f / Lsum;
        float x[4] = {acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv};
        const int r = rg * kRowsPerCta + rr;
        const int tq = r / a.group;
        const int h = kvh * a.group + (r - tq * a.group);
        *reinterpret_cast<float4*>(a.out + (((int64_t)b * a.q_len + tq) * a.num_q_heads + h) *
                                               kHeadDim + 4 * lane) =
            make_float4(x[0], x[1], x[2], x[3]);
    }
}

template <int BITS>
int stages_for()
{
    const int s = TQ_STAGE_BUDGET / Fmt<BITS>::kStageBytes;
    return s < 2 ? 2 : (s > kMaxStages ? kMaxStages : s);
}

template <int BITS>
size_t smem_for(int stages)
{
    const size_t ring = (size_t)kWarps * stages * Fmt<BITS>::kStageBytes;
    const size_t merge = (size_t)kWarps * kRowsPerCta * (kHeadDim + 2) * sizeof(float);
    return kRingOff + (ring > merge ? ring : merge);
}

template <int BITS, int NT>
cudaError_t launch_one(DecodeArgs a, dim3 grid, cudaStream_t stream)
{
    a.stages = stages_for<BITS>();
    const size_t smem = smem_for<BITS>(a.stages);
    static int configured_device_mask = 0;   // one bit per device ordinal < 31
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 31 || !(configured_device_mask & (1 << dev))) {
        e = cudaFuncSetAttribute(k_decode<BITS, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 31) configured_device_mask |= 1 << dev;
    }
    k_decode<BITS, NT><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

int decode_split_tokens(int page_size)
{
    return page_size >= 64 ? TQ_SPLIT_TOKENS_P64 : TQ_SPLIT_TOKENS;
}


int decode_tc_rows(int format, int G);
cudaError_t launch_decode_tc(const void* q, const tq_cache& c, int64_t block_bytes,
                             const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                             int batch, int q_len, int num_q_heads, int max_seq_len, float* out,
                             void* workspace, int split_tokens, cudaStream_t stream);

// Query rows per CTA: the tensor-core kernels (turbo formats) take 4, 8 or
// 16 (decode_tc_rows), the warp-MMA kernel (bf16) 8.
int decode_rows_per_cta(int format, int G)
{
    return format == 16 ? kRowsPerCta : decode_tc_rows(format, G);
}

int decode_row_groups(int format, int G)
{
    const int rows = decode_rows_per_cta(format, G);
    return (G + rows - 1) / rows;
}

// Workspace: [counters (256-byte aligned)][m,l partials][O partials]
bool decode_uses_prefill(int format, int G);

size_t decode_workspace_bytes(int batch, int num_kv_heads, int G, int max_seq_len, int page_size,
                              int format)
{
    if (decode_uses_prefill(format, G)) return 0;       // rows written directly
    const int st = decode_split_tokens(page_size);
    const int64_t max_splits = (max_seq_len + st - 1) / st;
    if (max_splits <= 1) return 0;
    const int rows = decode_rows_per_cta(format, G);
    const int64_t units = (int64_t)batch * num_kv_heads * decode_row_groups(format, G);
    const int64_t cnt = ((units * 4 + 255) / 256) * 256;
    const int64_t ml = ((units * max_splits * rows * 8 + 255) / 256) * 256;
    const int64_t ob = units * max_splits * rows * kHeadDim * 4;
    return (size_t)(cnt + ml + ob);
}

cudaError_t launch_decode(const void* q, const tq_cache& c, int64_t block_bytes,
                          const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                          int batch, int q_len, int num_q_heads, int max_seq_len, float* out,
                          void* workspace, cudaStream_t stream)
{
    if (c.format != 16)
        return launch_decode_tc(q, c, block_bytes, page_table, max_pages, seq_lens, batch, q_len,
                                num_q_heads, max_seq_len, out, workspace,
                                decode_split_tokens(c.page_size), stream);
    DecodeArgs a{};
    a.q = static_cast<const uint16_t*>(q);
    a.kv = static_cast<const uint8_t*>(c.pages);
    a.page_table = page_table;
    a.seq_lens = seq_lens;
    a.out = out;
    a.err = c.dev_error;
    a.block_bytes = block_bytes;
    a.max_pages = max_pages;
    a.num_pages = c.num_pages;
    a.num_kv_heads = c.num_kv_heads;
    a.num_q_heads = num_q_heads;
    a.group = num_q_heads / c.num_kv_heads;
    a.q_len = q_len;
    a.G = q_len * a.group;
    a.R = decode_row_groups(16, a.G);
    a.page_size = c.page_size;
    a.split_tokens = decode_split_tokens(c.page_size);
    a.max_splits = (max_seq_len + a.split_tokens - 1) / a.split_tokens;
    a.max_seq_len = max_seq_len;
    if (a.max_splits > 1) {
        const int64_t units = (int64_t)batch * c.num_kv_heads * a.R;
        const int64_t cnt = ((units * 4 + 255) / 256) * 256;
        const int64_t ml = ((units * a.max_splits * kRowsPerCta * 8 + 255) / 256) * 256;
        uint8_t* w = static_cast<uint8_t*>(workspace);
        a.ws_cnt = reinterpret_cast<uint32_t*>(w);
        a.ws_ml = reinterpret_cast<float2*>(w + cnt);
        a.ws_o = reinterpret_cast<float*>(w + cnt + ml);
    }
    const dim3 grid((unsigned)a.max_splits, (unsigned)(c.num_kv_heads * a.R), (unsigned)batch);
    const bool two = (a.G > 4);   // more than 4 rows in a row group
    return two ? launch_one<16, 2>(a, grid, stream) : launch_one<16, 1>(a, grid, stream);
}

}  // namespace tq
