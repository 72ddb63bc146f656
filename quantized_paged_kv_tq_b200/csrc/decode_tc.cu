// Paged decode / speculative-verify attention over a TurboQuant cache on the
// 5th-generation tensor cores (tcgen05, tensor memory).
//
// "xInfer: Pure-Rust LLM Inference Without a Python Runtime", section
// "TurboQuant is a memory trade": reading a low-bit KV cache dequantises on
// every attention step.  "infero", section "Continuous batching": a running
// batch shares the GPU over a paged KV cache.
//
// Two kernels share the structure below:
//   k_decode_i8  (2-, 4- and 8-bit codes, up to 8 query rows per kv head):
//                integer MMAs (kind::i8) on the codes as bytes; see the
//                section "Integer tensor-core variant" further down.
//   k_decode_tc  (3-bit codes, and any format with 9-16 rows per kv head):
//                f16 MMAs (kind::f16) on codes unpacked to exact f16
//                integers; described here.
//
// One CTA (128 threads) owns one (sequence, kv head, row group, split) with
// splits of 2048 tokens (1024 for 64-token pages) fixed by the sequence
// length alone.  The split is walked in tiles of 128 tokens; each page of a
// tile (its adjacent K and V blocks) arrives by one 1-D bulk async copy into
// a 2-stage ring.
// Per tile (k_decode_tc):
//   1. thread t unpacks token t's K codes into exact f16 integers and stores
//      them into tensor memory (lane t): the A operand of S = K q'.
//   2. one thread issues S[128 tok][N] = A x Q' (Q' in shared memory: the
//      rotated query, split into f16 hi and lo columns, N = 2 x rows).
//   3. thread t reads its token's scores from tensor memory (hi + lo), scales
//      them by s_k / L, and runs the online softmax (a lazy max: rescale only
//      when a tile beats the running max by 2^8; one CTA-wide vote per tile).
//      P' = p * s_v / L is written, split hi/lo in f16, to shared memory as
//      the B operand of the PV product.
//   4. thread d unpacks dimension d's V codes of the tile (the V block is
//      dim-major) into tensor memory (lane d): A operand of O^T += V^T P'.
//      The accumulator O^T lives in tensor memory for the whole split.
// The epilogue merges the split (last CTA of a sequence/kv head wins an
// atomic ticket and merges all splits), rotates back (H o / sqrt(d)) and
// writes fp32 output.
#include <algorithm>
#include <cstdint>
#include <math_constants.h>

#include "tq_device.cuh"

namespace tq {

namespace {

constexpr int kTcThreads = 128;
constexpr int kTile = 128;               // tokens per tile (= tensor-memory lanes)
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 128;      // A: 64 columns, S: N, O: N (N <= 32)
constexpr float kLog2eTc = 1.4426950408889634f;
constexpr float kLazyTc = 8.f;
constexpr uint32_t kPollsTc = 1u << 16;       // x 20 us sleeping polls
constexpr uint32_t kMagicTc = 0x64006400u;

struct TcArgs {
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
    int G;
    int R;             // row groups
    int page_size;
    int lp;            // log2(page_size)
    int split_tokens;
    int max_splits;
    int max_seq_len;
};

template <int BITS, bool FP8 = false>
struct TcFmt {
    static constexpr int CB = 16 * BITS;              // K row bytes (128 codes)
    static constexpr int L = (1 << (BITS - 1)) - 1;
    // codes come out of the unpacker in pairs (j, j + GB/2) of groups of GB
    // (E4M3 codes convert in adjacent pairs: GB = 2)
    static constexpr int GB = FP8 ? 2 : (BITS == 2 ? 16 : (BITS == 8 ? 4 : 8));
    static constexpr float kDequant = FP8 ? 1.f / 448.f : 1.f / (float)L;   // code -> value / s
    static constexpr int kStage = 2 * kTile * (CB + 4);   // K and V blocks of one tile
};

// Shared-memory header of the f16 kernel (byte offsets): barriers at 0,
// TMEM address and flags at 64, per-warp row reductions with a stride of kRS
// rows, the split's page ids, then the operands.  Up to 8 rows the header
// is 1 KB, so that three CTAs with two 33 KB stages of 8-bit codes fit the
// 228 KB of an SM.
template <int RG>
struct TcHdr {
    static constexpr int kRS = RG <= 8 ? 8 : 16;
    static constexpr int kRed = 128;                   // float [4][kRS]
    static constexpr int kRedv = kRed + 16 * kRS;      // unsigned [4]
    static constexpr int kRowfac = kRedv + 16;         // float [kRS]
    static constexpr int kL = kRowfac + 4 * kRS;       // float [4][kRS]
    static constexpr int kPid = RG <= 8 ? 512 : 1024;  // int [128]
    static constexpr int kBytes = kPid + 512;
    static_assert(RG <= kRS && kL + 16 * kRS <= kPid, "header overlap");
};

// Two E4M3 codes (low byte first) -> f16x2 (exact: every E4M3 value is an f16)
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t two)
{
    uint32_t d;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"((unsigned short)(two & 0xFFFFu)));
    return d;
}

// E4M3 K row (128 codes, chunks permuted as for 8-bit codes) -> tensor
// memory columns [0, 64), codes in order: column j holds codes 2j, 2j + 1.
__device__ __forceinline__ void k_row_to_tmem_fp8(const uint8_t* row, uint32_t taddr, int sw)
{
    uint32_t o[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 a = *reinterpret_cast<const uint4*>(row + 16 * ((2 * q) ^ sw));
        const uint4 b = *reinterpret_cast<const uint4*>(row + 16 * ((2 * q + 1) ^ sw));
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            o[2 * i] = e4m3x2_f16x2(w[i]);
            o[2 * i + 1] = e4m3x2_f16x2(w[i] >> 16);
        }
        tmem_st16(taddr + 16 * q, o);
    }
}

// f16 NaN lanes -> 65504 (min.f16x2 returns the other operand of a NaN).
// The encoder saturates, so a cached E4M3 code is never NaN; stage bytes past
// the end of a sequence may be, and their zero weights must give zero products.
__device__ __forceinline__ uint32_t finite_f16x2(uint32_t h)
{
    uint32_t d;
    asm("min.f16x2 %0, %1, %2;" : "=r"(d) : "r"(h), "r"(0x7BFF7BFFu));
    return d;
}

// E4M3 V codes of dimension `dim` for the tile's 128 tokens -> tensor memory
// columns [0, 64) of this lane, tokens in order (vblk0, bb as v_col_to_tmem).
__device__ __forceinline__ void v_col_to_tmem_fp8(const uint8_t* vblk0, int64_t bb, int lp,
                                                  int dim, uint32_t taddr)
{
    const int P = 1 << lp;
    uint32_t o[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int t0 = 32 * q, pg = t0 >> lp, in = t0 & (P - 1);
        const uint8_t* row = vblk0 + pg * bb + (int64_t)dim * P;
        uint4 x, y;
        if (P >= 32) {
            x = *reinterpret_cast<const uint4*>(row + in);
            y = *reinterpret_cast<const uint4*>(row + in + 16);
        } else {
            x = *reinterpret_cast<const uint4*>(row);
            y = *reinterpret_cast<const uint4*>(row + bb);
        }
        const uint32_t w[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            o[2 * i] = finite_f16x2(e4m3x2_f16x2(w[i]));
            o[2 * i + 1] = finite_f16x2(e4m3x2_f16x2(w[i] >> 16));
        }
        tmem_st16(taddr + 16 * q, o);
    }
}

// Index (dimension for K, token for V) held at K position k of an A operand,
// i.e. the order the unpacker emits: pair c holds (perm(2c), perm(2c + 1)).
template <int GB>
__device__ __forceinline__ int perm_k(int k)
{
    return (k / GB) * GB + ((k % GB) >> 1) + (GB / 2) * (k & 1);
}
template <int GB>
__device__ __forceinline__ int perm_inv(int i)
{
    const int m = i % GB;
    return (i / GB) * GB + (m < GB / 2 ? 2 * m : 2 * (m - GB / 2) + 1);
}

// f16x2 of (code a, code b) from magic-number halves: (1024 + 2^s u) * 2^-s - (1024 2^-s + L)
__device__ __forceinline__ uint32_t mk(uint32_t bits_with_magic, uint32_t mul, uint32_t add)
{
    return hfma2_u32(bits_with_magic, mul, add);
}

// ---------------------------------------------------------------- unpack
// Emit the pairs of one 32-bit word of 4-bit codes (8 codes): (0,4) (1,5) (2,6) (3,7).
__device__ __forceinline__ void pairs4(uint32_t w, uint32_t* o)
{
    const uint32_t w8 = w >> 8;
    o[0] = mk(and_or(w, 0x000F000Fu, kMagicTc), 0x3C003C00u, 0xE407E407u);
    o[1] = mk(and_or(w, 0x00F000F0u, kMagicTc), 0x2C002C00u, 0xD470D470u);
    o[2] = mk(and_or(w8, 0x000F000Fu, kMagicTc), 0x3C003C00u, 0xE407E407u);
    o[3] = mk(and_or(w8, 0x00F000F0u, kMagicTc), 0x2C002C00u, 0xD470D470u);
}
// 8-bit codes (4 per word): (0,2) (1,3)
__device__ __forceinline__ void pairs8(uint32_t w, uint32_t* o)
{
    o[0] = mk(prmt(w, 0x64646464u, 0x4240u), 0x3C003C00u, 0xE47FE47Fu);
    o[1] = mk(prmt(w, 0x64646464u, 0x4341u), 0x3C003C00u, 0xE47FE47Fu);
}
// 2-bit codes (16 per word): (j, j+8), j = 0..7
__device__ __forceinline__ void pairs2(uint32_t w, uint32_t* o)
{
    constexpr uint32_t mul[4] = {0x3C003C00u, 0x34003400u, 0x2C002C00u, 0x24002400u};
    constexpr uint32_t add[4] = {0xE401E401u, 0xDC04DC04u, 0xD410D410u, 0xCC40CC40u};
    const uint32_t w8 = w >> 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int jj = j & 3;
        o[j] = mk(and_or(j < 4 ? w : w8, 0x00030003u << (2 * jj), kMagicTc), mul[jj], add[jj]);
    }
}
// 3-bit codes: one 24-bit group of 8 codes (bits 0..23 of g): (k, k+4), k = 0..3
__device__ __forceinline__ void pairs3(uint32_t g, uint32_t* o)
{
    constexpr uint32_t mul[3] = {0x3C003C00u, 0x30003000u, 0x24002400u};
    constexpr uint32_t add[3] = {0xE403E403u, 0xD818D818u, 0xCCC0CCC0u};
    const uint32_t sel = bitsel(g, g << 4, 0x0000FFFFu);
    const uint32_t sel3 = bitsel(g >> 3, g << 1, 0x0000FFFFu);
    o[0] = mk(and_or(sel, 0x00070007u, kMagicTc), mul[0], add[0]);
    o[1] = mk(and_or(sel, 0x00380038u, kMagicTc), mul[1], add[1]);
    o[2] = mk(and_or(sel, 0x01C001C0u, kMagicTc), mul[2], add[2]);
    o[3] = mk(and_or(sel3, 0x01C001C0u, kMagicTc), mul[2], add[2]);
}

// K row of one token (128 codes; 16-byte chunks permuted by `sw`, see
// k_swizzle) as 64 words of f16 pairs, handed to sink(c, o) 16 words at a
// time (words c .. c + 15).
template <int BITS, class Sink>
__device__ __forceinline__ void k_row_unpack(const uint8_t* row, int sw, Sink&& sink)
{
    uint32_t o[16];
    auto chunk = [&](int c) { return *reinterpret_cast<const uint4*>(row + 16 * (c ^ sw)); };
    if constexpr (BITS == 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 w = chunk(q);
            pairs4(w.x, o);
            pairs4(w.y, o + 4);
            pairs4(w.z, o + 8);
            pairs4(w.w, o + 12);
            sink(16 * q, o);
        }
    } else if constexpr (BITS == 8) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 a = chunk(2 * q);
            const uint4 b = chunk(2 * q + 1);
            pairs8(a.x, o); pairs8(a.y, o + 2); pairs8(a.z, o + 4); pairs8(a.w, o + 6);
            pairs8(b.x, o + 8); pairs8(b.y, o + 10); pairs8(b.z, o + 12); pairs8(b.w, o + 14);
            sink(16 * q, o);
        }
    } else if constexpr (BITS == 2) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint4 w = chunk(q);
            pairs2(w.x, o);
            pairs2(w.y, o + 8);
            sink(32 * q, o);
            pairs2(w.z, o);
            pairs2(w.w, o + 8);
            sink(32 * q + 16, o);
        }
    } else {  // 3 bits: 48-byte row, 12 words, 16 groups of 8 codes
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            // 12 bytes = 3 words = 4 groups
            const uint32_t* p = reinterpret_cast<const uint32_t*>(row + 12 * q);
            const uint32_t W0 = p[0], W1 = p[1], W2 = p[2];
            pairs3(W0, o);
            pairs3(prmt(W0, W1, 0x6543u), o + 4);
            pairs3(prmt(W1, W2, 0x5432u), o + 8);
            pairs3(W2 >> 8, o + 12);
            sink(16 * q, o);
        }
    }
}

// ... into tensor memory columns [0, 64) of this thread's lane
template <int BITS>
__device__ __forceinline__ void k_row_to_tmem(const uint8_t* row, uint32_t taddr, int sw)
{
    k_row_unpack<BITS>(row, sw, [&](int c, const uint32_t* o) { tmem_st16(taddr + c, o); });
}

// V codes of dimension `dim` for the 128 tokens of a tile as 64 words of
// f16 pairs, handed to sink(c, o) 16 words at a time.  vblk0: V block of the
// tile's first page in the stage; the V blocks of later pages follow every
// `bb` bytes.
template <int BITS, class Sink>
__device__ __forceinline__ void v_col_unpack(const uint8_t* vblk0, int64_t bb, int lp, int dim,
                                             Sink&& sink)
{
    const int P = 1 << lp;
    uint32_t o[16];
    // tokens are emitted 16 pairs (32 tokens) per store
    const int row_bytes = P * BITS / 8;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int t0 = 32 * q;                   // first tile token of this chunk
        const int pg = t0 >> lp;                 // page holding it
        const int in = t0 & (P - 1);             // its offset in the page
        const uint8_t* row = vblk0 + pg * bb + (int64_t)dim * row_bytes;
        if constexpr (BITS == 4) {
            // 32 tokens = 16 bytes of one row (P >= 32) or two 8-byte rows (P = 16)
            uint32_t w[4];
            if (P >= 32) {
                const uint4 x = *reinterpret_cast<const uint4*>(row + in / 2);
                w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
            } else {
                const uint2 x = *reinterpret_cast<const uint2*>(row);
                const uint2 y = *reinterpret_cast<const uint2*>(row + bb);
                w[0] = x.x; w[1] = x.y; w[2] = y.x; w[3] = y.y;
            }
            pairs4(w[0], o); pairs4(w[1], o + 4); pairs4(w[2], o + 8); pairs4(w[3], o + 12);
        } else if constexpr (BITS == 8) {
            // 32 tokens = 32 bytes (P >= 32) or two 16-byte rows (P = 16)
            uint4 x, y;
            if (P >= 32) {
                x = *reinterpret_cast<const uint4*>(row + in);
                y = *reinterpret_cast<const uint4*>(row + in + 16);
            } else {
                x = *reinterpret_cast<const uint4*>(row);
                y = *reinterpret_cast<const uint4*>(row + bb);
            }
            pairs8(x.x, o); pairs8(x.y, o + 2); pairs8(x.z, o + 4); pairs8(x.w, o + 6);
            pairs8(y.x, o + 8); pairs8(y.y, o + 10); pairs8(y.z, o + 12); pairs8(y.w, o + 14);
        } else if constexpr (BITS == 2) {
            // 32 tokens = 8 bytes (P >= 32) or two 4-byte rows (P = 16)
            uint32_t a, c;
            if (P >= 32) {
                const uint2 x = *reinterpret_cast<const uint2*>(row + in / 4);
                a = x.x; c = x.y;
            } else {
                a = *reinterpret_cast<const uint32_t*>(row);
                c = *reinterpret_cast<const uint32_t*>(row + bb);
            }
            pairs2(a, o);
            pairs2(c, o + 8);
        } else {
            // 3 bits: 16 tokens are 6 bytes at a 2-byte boundary of the block;
            // read the two aligned words around them and shift
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // 16 tokens from a longer page, or the whole next 16-token page
                const int tk = (P >= 32) ? in + 16 * h : 0;    // first token in its page
                const int hp = (P >= 32) ? pg : pg + h;        // page of these 16
                const int off = dim * row_bytes + 3 * tk / 8;  // byte offset in block
                const uint32_t* wp =
                    reinterpret_cast<const uint32_t*>(vblk0 + hp * bb + (off & ~3));
                const uint64_t v64 = (((uint64_t)wp[1] << 32) | wp[0]) >> ((off & 3) * 8);
                pairs3((uint32_t)v64 & 0xFFFFFFu, o + 8 * h);
                pairs3((uint32_t)(v64 >> 24) & 0xFFFFFFu, o + 8 * h + 4);
            }
        }
        sink(16 * q, o);
    }
}

// ... into tensor memory columns [0, 64) of this thread's lane
template <int BITS>
__device__ __forceinline__ void v_col_to_tmem(const uint8_t* vblk0, int64_t bb, int lp, int dim,
                                              uint32_t taddr)
{
    v_col_unpack<BITS>(vblk0, bb, lp, dim,
                       [&](int c, const uint32_t* o) { tmem_st16(taddr + c, o); });
}

// Bulk copies of one tile's pages into a stage (warp 0): one copy per page of
// its adjacent K and V blocks, so the stage is [page][K block, V block].
// pids[j]: physical page of the tile's j-th page (global page table or the
// split's copy in shared memory).
__device__ __forceinline__ void issue_tile_tc(uint8_t* stage, uint64_t* bar, const TcArgs& a,
                                              const int* pids, int kvh, int ntok, int lane)
{
    const int npg = (ntok + (1 << a.lp) - 1) >> a.lp;     // pages holding tokens
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(2 * npg * a.block_bytes));
    __syncwarp();
    if (lane < npg) {
        int pid = pids[lane];
        if (pid < 0 || pid >= a.num_pages) {
            report_error(a.err, TQ_ERR_DEVICE_CHECK, kErrPageRange);
            pid = 0;
        }
        const int64_t off = ((int64_t)pid * a.num_kv_heads + kvh) * 2 * a.block_bytes;
        bulk_g2s(stage + lane * 2 * a.block_bytes, a.kv + off, (uint32_t)(2 * a.block_bytes), bar);
    }
}

// The same copies spread over warps 1..3 (warp 0 issues S = K q'' at that
// point): warp w takes pages w - 1, w + 2, w + 5, ...; each warp's lane 0
// arrives with its own byte count (the stage barrier counts 4 arrivals, warp
// 0 with none), so no warp waits on another to issue.
__device__ __forceinline__ void issue_tile_warps(uint8_t* stage, uint64_t* bar, const TcArgs& a,
                                                 const int* pids, int kvh, int ntok, int warp,
                                                 int lane)
{
    const int npg = (ntok + (1 << a.lp) - 1) >> a.lp;
    const int first = warp - 1;
    const int mine = (warp > 0 && npg > first) ? (npg - first + 2) / 3 : 0;   // pages of this warp
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(2 * mine * a.block_bytes));
    __syncwarp();
    if (lane < mine) {
        const int j = first + 3 * lane;
        int pid = pids[j];
        if (pid < 0 || pid >= a.num_pages) {
            report_error(a.err, TQ_ERR_DEVICE_CHECK, kErrPageRange);
            pid = 0;
        }
        const int64_t off = ((int64_t)pid * a.num_kv_heads + kvh) * 2 * a.block_bytes;
        bulk_g2s(stage + j * 2 * a.block_bytes, a.kv + off, (uint32_t)(2 * a.block_bytes), bar);
    }
}

// The split's page ids -> shared memory (at most 128: 2048 tokens of 16).
__device__ __forceinline__ void load_split_pids(int* s_pid, const TcArgs& a, int b, int tok_begin,
                                                int tok_end, int tid)
{
    const int first = tok_begin >> a.lp;
    const int n = ((tok_end - 1) >> a.lp) - first + 1;
    if (tid < n) s_pid[tid] = __ldg(a.page_table + (int64_t)b * a.max_pages + first + tid);
}

// Split epilogue shared by the tensor-core kernels.  sO: the split's
// un-normalised output rows [RG][128] (rotated domain); s_l: per-warp partial
// row sums [4][LS]; m_run: row maxima (log2 units).  A split that is the whole
// sequence normalises, rotates back and writes; otherwise the partial goes to
// the workspace and the last split CTA of the unit (atomic ticket) merges;
// `unit` indexes the (sequence, kv head, row group) in the workspace.
// valid == false (the CTA gave up on a bounded wait; CTA-uniform): nothing
// is read from sO, s_l or m_run; a split of a longer sequence still records
// an empty partial (m = -inf) and takes its ticket, so the unit's counter
// wraps back to zero and the workspace stays usable for later calls.
template <int RG, int LS, bool ROT = true>
__device__ __forceinline__ void tc_finish(const TcArgs& a, const float* sO, const float* s_l,
                                          const float* m_run, int* s_flag, int b, int kvh, int rg,
                                          int split, int nsplit, int nrows, int warp, int lane,
                                          int tid, bool valid, int64_t unit)
{
    const int64_t part = unit * a.max_splits + split;
    const float rs = 0.08838834764831845f;
    if (!valid && nsplit == 1) return;
    for (int rr = warp; rr < nrows; rr += 4) {
        if (!valid) {
            if (lane == 0) a.ws_ml[part * RG + rr] = make_float2(-CUDART_INF_F, 0.f);
            continue;
        }
        const float M = m_run[rr];
        const float Lsum = s_l[rr] + s_l[LS + rr] + s_l[2 * LS + rr] + s_l[3 * LS + rr];
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = sO[rr * kHeadDim + 4 * lane + e];
        const int R = rg * RG + rr;
        const int tq = R / a.group;
        const int h = kvh * a.group + (R - tq * a.group);
        if (nsplit == 1) {
            const float inv = 1.f / Lsum;
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] *= inv;
            if (ROT) fwht128_lane(x, lane);
            const float sc = ROT ? rs : 1.f;
            *reinterpret_cast<float4*>(a.out + (((int64_t)b * a.q_len + tq) * a.num_q_heads + h) *
                                                   kHeadDim + 4 * lane) =
                make_float4(x[0] * sc, x[1] * sc, x[2] * sc, x[3] * sc);
        } else {
            *reinterpret_cast<float4*>(a.ws_o + (part * RG + rr) * kHeadDim + 4 * lane) =
                make_float4(x[0], x[1], x[2], x[3]);
            if (lane == 0) a.ws_ml[part * RG + rr] = make_float2(M, Lsum);
        }
    }
    if (nsplit == 1) return;

    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned old = atomicInc(a.ws_cnt + unit, (unsigned)(nsplit - 1));
        s_flag[1] = old == (unsigned)(nsplit - 1);
    }
    __syncthreads();
    if (!s_flag[1]) return;
    __threadfence();
    for (int rr = warp; rr < nrows; rr += 4) {
        const int64_t base = unit * a.max_splits;
        float M = -CUDART_INF_F;
        for (int sp = 0; sp < nsplit; ++sp)
            M = fmaxf(M, __ldcg(a.ws_ml + (base + sp) * RG + rr).x);
        float Lsum = 0.f;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int sp = 0; sp < nsplit; ++sp) {
            const float2 ml = __ldcg(a.ws_ml + (base + sp) * RG + rr);
            if (ml.x == -CUDART_INF_F) continue;       // empty split: no keys, no O written
            const float sc = exp2f(ml.x - M);
            Lsum += sc * ml.y;
            const float4 v = __ldcg(reinterpret_cast<const float4*>(
                a.ws_o + ((base + sp) * RG + rr) * kHeadDim) + lane);
            acc[0] += sc * v.x;
            acc[1] += sc * v.y;
            acc[2] += sc * v.z;
            acc[3] += sc * v.w;
        }
        const float inv = 1.f / Lsum;
        float x[4] = {acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv};
        if (ROT) fwht128_lane(x, lane);
        const float sc = ROT ? rs : 1.f;
        const int R = rg * RG + rr;
        const int tq = R / a.group;
        const int h = kvh * a.group + (R - tq * a.group);
        *reinterpret_cast<float4*>(a.out + (((int64_t)b * a.q_len + tq) * a.num_q_heads + h) *
                                               kHeadDim + 4 * lane) =
            make_float4(x[0] * sc, x[1] * sc, x[2] * sc, x[3] * sc);
    }
}

// FP8: E4M3 codes (BITS = 8 layout), converted to f16; no rotation of the
// query or of the output.
template <int BITS, int RG, bool FP8 = false>
__global__ void __launch_bounds__(kTcThreads, 4)
k_decode_tc(const TcArgs a)
{
    using F = TcFmt<BITS, FP8>;
    // RG query rows per CTA; operand columns: hi parts [0, RG), lo parts
    // [RG, 2 RG), zero padding up to NCOL (the MMA needs N >= 16)
    constexpr int NCOL = 2 * RG < 16 ? 16 : 2 * RG;
    constexpr uint32_t kColS = 64, kColO = 64 + NCOL;
    // instruction descriptors: f32 accumulate, f16 operands, M = 128, N = NCOL;
    // B K-major (Q') for S, B MN-major (P') for O
    constexpr uint32_t kIdescS = (1u << 4) | ((uint32_t)(NCOL >> 3) << 17) | (8u << 24);
    constexpr uint32_t kIdescO = kIdescS | (1u << 16);
    constexpr uint32_t kCmRow = (NCOL / 8) * 128;   // bytes per 8-deep K group

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);              // [kStages]
    uint64_t* bar_s = full + kStages;
    uint64_t* bar_o = bar_s + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + 64);
    int* s_flag = reinterpret_cast<int*>(smem + 68);                 // [0] abort, [1] ticket
    using H = TcHdr<RG>;
    float* s_red = reinterpret_cast<float*>(smem + H::kRed);         // [4][kRS] row maxima
    unsigned* s_redv = reinterpret_cast<unsigned*>(smem + H::kRedv); // [4]
    float* s_rowfac = reinterpret_cast<float*>(smem + H::kRowfac);   // [kRS]
    float* s_l = reinterpret_cast<float*>(smem + H::kL);             // [4][kRS]
    int* s_pid = reinterpret_cast<int*>(smem + H::kPid);             // [128] split page ids
    uint8_t* s_qb = smem + H::kBytes;                                // Q' operand
    uint8_t* s_pb = s_qb + 256 * NCOL;                               // P' operand / q staging
    uint8_t* ring = s_pb + 256 * NCOL;

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

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tok_begin = split * a.split_tokens;
    const int tok_end = min(seq_len, tok_begin + a.split_tokens);
    const int ntiles = (tok_end - tok_begin + kTile - 1) / kTile;
    const int P = a.page_size;

    // ---- set-up: barriers, tensor memory, first copies
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        s_flag[0] = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * warp) << 16);   // this thread's lane

    if (warp == 0) {
        for (int s = 0; s < kStages && s < ntiles; ++s) {
            const int t0 = tok_begin + s * kTile;
            issue_tile_tc(ring + s * F::kStage, &full[s], a,
                          a.page_table + (int64_t)b * a.max_pages + (t0 >> a.lp), kvh,
                          min(kTile, tok_end - t0), lane);
        }
    }

    load_split_pids(s_pid, a, b, tok_begin, tok_end, tid);   // visible after the next barrier

    // ---- query rows of this row group: rotate, scale to log2 units,
    // power-of-two prescale (hi and lo parts stay normal f16)
    float* s_qf = reinterpret_cast<float*>(s_pb);                    // [RG][128]
    for (int rr = warp; rr < RG; rr += 4) {
        const int r = rg * RG + rr;
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
        if (!FP8) fwht128_lane(x, lane);
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // turbo: (H q / sqrt d) . y / sqrt d = (H q) . y / d; fp8: q . x / sqrt d
            x[e] *= FP8 ? kLog2eTc * 0.08838834764831845f : kLog2eTc / kHeadDim;
            amax = fmaxf(amax, fabsf(x[e]));
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, m));
        const int ex = amax > 0.f ? max(-100, min(100, ilogbf(amax))) : 0;
        const float pre = pow2i(12 - ex);
#pragma unroll
        for (int e = 0; e < 4; ++e) s_qf[rr * kHeadDim + 4 * lane + e] = x[e] * pre;
        if (lane == 0) s_rowfac[rr] = pow2i(ex - 12);
    }
    __syncthreads();
    {
        // Q' operand, K-major: K position k = tid holds dimension perm(k);
        // column n < RG is row n's hi part, n >= RG its lo part
        const int k = tid;
        const int dim = perm_k<F::GB>(k);
        __half* qb = reinterpret_cast<__half*>(s_qb);
#pragma unroll
        for (int n = 0; n < NCOL; ++n) {
            const float v = n < 2 * RG ? s_qf[(n % RG) * kHeadDim + dim] : 0.f;
            const float hi = __half2float(__float2half_rn(v));
            const __half h = __float2half_rn(n < RG ? v : v - hi);
            const int cm = (k >> 3) * (NCOL / 8) + (n >> 3);
            qb[(cm * 128 + (n & 7) * 16 + (k & 7) * 2) / 2] = h;
        }
    }
    float rowfac[RG];
    int lim[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        rowfac[r] = s_rowfac[r];
        const int R = rg * RG + r;
        lim[r] = R < a.G ? seq_len - a.q_len + R / a.group : -1;
    }
    __syncthreads();   // the q staging (aliasing the P' buffer) is consumed
    if (2 * RG < NCOL) {
        // zero padding columns of the P' operand, written once
        uint8_t* rowp = s_pb + (tid >> 3) * kCmRow + (tid & 7) * 16;
#pragma unroll
        for (int ng = 2 * RG / 8; ng < NCOL / 8; ++ng)
            *reinterpret_cast<uint4*>(rowp + ng * 128) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    __syncthreads();
    const uint64_t desc_q = smem_desc(s_qb, kCmRow, 128);
    const uint64_t desc_p = smem_desc(s_pb, kCmRow, 128);

    float m_run[RG], l_run[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        m_run[r] = -CUDART_INF_F;
        l_run[r] = 0.f;
    }
    int ev = 0;                                   // running V-scale exponent (biased)
    float vn = 1.f;                               // 2^(127 - ev)
    float vlimit = __uint_as_float(1u << 23);     // scales >= this raise ev
    const float kinv = F::kDequant;
    const int lim_min = seq_len - a.q_len + (rg * RG) / a.group;
    const int kpos = perm_inv<F::GB>(tid);        // this token's K position in PV
    bool aborted = false;

    for (int tt = 0; tt < ntiles; ++tt) {
        const int stage = tt % kStages;
        uint8_t* st = ring + stage * F::kStage;
        const int tok0 = tok_begin + tt * kTile;
        bool ok = mbar_wait_sleep(&full[stage], (uint32_t)((tt / kStages) & 1), kPollsTc);
        if (tt > 0) ok = ok && mbar_wait_sleep(bar_o, (uint32_t)((tt - 1) & 1), kPollsTc);
        tc_fence_after();
        if (!ok) atomicOr(&s_flag[0], 1);

        // 1. K row of token tid -> A operand
        const int pg = tid >> a.lp, row = tid & (P - 1);
        const uint8_t* kblk = st + pg * 2 * a.block_bytes;     // stage: [page][K block, V block]
        const uint8_t* vblk = kblk + a.block_bytes;
        if constexpr (FP8) k_row_to_tmem_fp8(kblk + row * F::CB, t_lane, k_swizzle<8>(row));
        else k_row_to_tmem<BITS>(kblk + row * F::CB, t_lane, k_swizzle<BITS>(row));
        float ks = reinterpret_cast<const float*>(kblk + P * F::CB)[row] * kinv;
        float vs = reinterpret_cast<const float*>(vblk + P * F::CB)[row] * kinv;
        const int tok = tok0 + tid;
        if (tok >= tok_end) { ks = 0.f; vs = 0.f; }       // slot never written
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (s_flag[0]) { aborted = true; break; }

        // 2. S = K Q'
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                umma_f16_ts(tmem + kColS, tmem + 8 * j, desc_q + ((2 * j * kCmRow) >> 4), kIdescS,
                            j > 0);
            umma_commit(bar_s);
        }
        ok = mbar_wait_sleep(bar_s, (uint32_t)(tt & 1), kPollsTc);
        tc_fence_after();
        if (!ok) atomicOr(&s_flag[0], 1);

        // 3. scores of token tid; V column of dimension tid -> A operand
        uint32_t sraw[NCOL];
#pragma unroll
        for (int c = 0; c < NCOL; c += 16) tmem_ld16(t_lane + kColS + c, sraw + c);
        if constexpr (FP8) v_col_to_tmem_fp8(st + a.block_bytes, 2 * a.block_bytes, a.lp, tid, t_lane);
        else v_col_to_tmem<BITS>(st + a.block_bytes, 2 * a.block_bytes, a.lp, tid, t_lane);
        tmem_wait_ld();
        const bool full_tile = tok0 + kTile - 1 <= lim_min;
        float sc[RG];
        bool need = false;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            float x = (__uint_as_float(sraw[r]) + __uint_as_float(sraw[RG + r])) * (ks * rowfac[r]);
            if (!full_tile) x = tok <= lim[r] ? x : -CUDART_INF_F;
            sc[r] = x;
            need |= x > m_run[r] + kLazyTc;
        }
        need |= vs >= vlimit;
        const int any = __syncthreads_or(need);          // also: the stage is consumed
        if (s_flag[0]) { aborted = true; break; }
        if (warp == 0 && tt + kStages < ntiles) {
            const int t0 = tok_begin + (tt + kStages) * kTile;
            issue_tile_tc(st, &full[stage], a, s_pid + ((t0 - tok_begin) >> a.lp), kvh,
                          min(kTile, tok_end - t0), lane);
        }
        if (any) {
            // exact tile maxima of every row and of the V scales
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                float v = sc[r];
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
                if (lane == 0) s_red[warp * H::kRS + r] = v;
            }
            const unsigned vb = __reduce_max_sync(kFull, __float_as_uint(vs));
            if (lane == 0) s_redv[warp] = vb;
            __syncthreads();
            const unsigned vmax = max(max(s_redv[0], s_redv[1]), max(s_redv[2], s_redv[3]));
            const int ev_new = max(ev, (int)(vmax >> 23));
            const float av = pow2i(ev - ev_new);
            ev = ev_new;
            vn = pow2i(127 - ev);
            vlimit = ev >= 254 ? CUDART_INF_F : __uint_as_float((uint32_t)(ev + 1) << 23);
            float alpha[RG];
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                const float tmax = fmaxf(fmaxf(s_red[r], s_red[H::kRS + r]),
                                         fmaxf(s_red[2 * H::kRS + r], s_red[3 * H::kRS + r]));
                const float mn = fmaxf(m_run[r], tmax);
                alpha[r] = mn == -CUDART_INF_F ? 1.f : fast_exp2(m_run[r] - mn);
                m_run[r] = mn;
                l_run[r] *= alpha[r];
            }
            if (tt > 0) {
                // O^T row (dimension tid): column n holds row n % RG
                uint32_t ov[NCOL];
#pragma unroll
                for (int c = 0; c < NCOL; c += 16) tmem_ld16(t_lane + kColO + c, ov + c);
                tmem_wait_ld();
#pragma unroll
                for (int n = 0; n < NCOL; ++n)
                    ov[n] = __float_as_uint(__uint_as_float(ov[n]) * (alpha[n % RG] * av));
#pragma unroll
                for (int c = 0; c < NCOL; c += 16) tmem_st16(t_lane + kColO + c, ov + c);
            }
            __syncthreads();   // s_red is reused by the next rescale
        }

        // P' row of token tid at K position kpos: hi columns, then lo columns
        const float vn_t = vs * vn;
        uint32_t hl[RG];          // half2 pairs: hi parts [0, RG/2), lo parts [RG/2, RG)
        uint32_t* hv = hl;
        uint32_t* lv = hl + RG / 2;
#pragma unroll
        for (int r = 0; r < RG; r += 2) {
            float p0 = fast_exp2(sc[r] - m_run[r]);
            float p1 = fast_exp2(sc[r + 1] - m_run[r + 1]);
            if (!full_tile) {
                p0 = sc[r] == -CUDART_INF_F ? 0.f : p0;
                p1 = sc[r + 1] == -CUDART_INF_F ? 0.f : p1;
            }
            l_run[r] += p0;
            l_run[r + 1] += p1;
            float x0 = p0 * vn_t, x1 = p1 * vn_t;
            if (!full_tile) {
                x0 = p0 > 0.f ? x0 : 0.f;
                x1 = p1 > 0.f ? x1 : 0.f;
            }
            hv[r / 2] = split_hi_lo<true>(x0, x1, true);
            lv[r / 2] = split_hi_lo<true>(x0, x1, false);
        }
        {
            uint8_t* rowp = s_pb + (kpos >> 3) * kCmRow + (kpos & 7) * 16;
#pragma unroll
            for (int ng = 0; ng < 2 * RG / 8; ++ng)
                *reinterpret_cast<uint4*>(rowp + ng * 128) =
                    make_uint4(hl[4 * ng], hl[4 * ng + 1], hl[4 * ng + 2], hl[4 * ng + 3]);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // 4. O^T += V^T P'
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                umma_f16_ts(tmem + kColO, tmem + 8 * j, desc_p + ((2 * j * kCmRow) >> 4), kIdescO,
                            (tt > 0 || j > 0) ? 1u : 0u);
            umma_commit(bar_o);
        }
    }

    // ---- epilogue: O rows into shared memory, l summed over the CTA.  The
    // decision to finish is taken for the whole CTA (warp-collective tensor
    // memory loads and the barriers of tc_finish follow).
    bool ok = !aborted && mbar_wait_sleep(bar_o, (uint32_t)((ntiles - 1) & 1), kPollsTc);
    tc_fence_after();
    ok = __syncthreads_and(ok);
    const int nrows = min(RG, a.G - rg * RG);
    float* sO = reinterpret_cast<float*>(ring);          // [RG][128]
    if (ok) {
        uint32_t ov[NCOL];
#pragma unroll
        for (int c = 0; c < NCOL; c += 16) tmem_ld16(t_lane + kColO + c, ov + c);
        tmem_wait_ld();
        const float vback = pow2i(ev - 127);
#pragma unroll
        for (int r = 0; r < RG; ++r)
            sO[r * kHeadDim + tid] = (__uint_as_float(ov[r]) + __uint_as_float(ov[RG + r])) * vback;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            float l = l_run[r];
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) l += __shfl_xor_sync(kFull, l, m);
            if (lane == 0) s_l[warp * H::kRS + r] = l;
        }
    } else if (tid == 0) {
        report_error(a.err, TQ_ERR_TIMEOUT, kErrWaitTile);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    tc_finish<RG, H::kRS, !FP8>(a, sO, s_l, m_run, s_flag, b, kvh, rg, split, nsplit, nrows, warp, lane,
                        tid, ok, (int64_t)b * gridDim.y + blockIdx.y);
}

// ===================================================================
// Integer tensor-core variant (kind::i8) for 2-, 4- and 8-bit codes.
//
//   S = K q''   A: K codes in tensor memory as unsigned bytes f_k u: a code
//               keeps its bit position inside its byte (f_k = 1 or 16 for the
//               low / high nibble of 4-bit codes; 1, 4, 16 or 64 for the
//               four 2-bit fields), so unpacking costs one AND per word.
//               B: (F / f_k) q'' with q'' = rint(q' 2^s) the fixed-point
//               rotated query, as four balanced signed byte digits per row
//               (column 4 r + d).  The accumulator starts at
//               -L sum_k f_k B[k], so digit column d ends as the exact
//               integer F sum_k (u_k - L) digit_d(q''_k) (|.| < 2^22).
//   O^T += V^T P''  A: V codes as unsigned bytes u (dim-major rows).
//               B: P'' = rint(p s_v / L 2^(127 - ev) 2^22) as four unsigned
//               byte digits per row.  O holds sum_t u_t P''_t exactly in
//               int32; the offset L sum_t P''_t is tracked exactly per row
//               (64-bit) and taken off in 64-bit integers when O is folded
//               into fp32 registers (on a rescale and at the end of the
//               split), so the fold rounds once.
// ===================================================================
template <int BITS>
struct I8Fmt {
    static constexpr int CB = 16 * BITS;
    static constexpr int L = (1 << (BITS - 1)) - 1;
    static constexpr int F = BITS == 4 ? 16 : (BITS == 2 ? 64 : 1);
    static constexpr int kStage = 2 * kTile * (CB + 4);
};

// CTAs per SM of the integer kernel: tensor memory holds 4 (128 columns
// each); with 4 query rows and 2- or 4-bit codes a fifth fits in registers
// (96) and shared memory, stages its first tiles and query operand, and waits
// in tcgen05.alloc until a running CTA frees its columns.
constexpr int i8_ctas_per_sm(int bits, int rg) { return (rg <= 4 && bits != 8) ? 5 : 4; }

// Shared-memory header of the integer kernel (bytes from the start).
constexpr int kI8Pid = 1024;        // [128] split page ids
constexpr int kI8Ps = 1536;         // [4][16] per-warp sums of P'' (u64)
constexpr int kI8Hdr = 2048;        // operands and the ring follow

// K position k of the byte operands -> dimension (K) or token (V)
template <int BITS>
__device__ __forceinline__ int perm_i8(int k)
{
    if constexpr (BITS == 4) return 8 * (k >> 3) + 2 * (k & 3) + ((k & 7) >> 2);
    if constexpr (BITS == 2) return 16 * (k >> 4) + 4 * (k & 3) + ((k & 15) >> 2);
    return k;
}
template <int BITS>
__device__ __forceinline__ int perm_i8_inv(int i)
{
    if constexpr (BITS == 4) return 8 * (i >> 3) + ((i & 7) >> 1) + 4 * (i & 1);
    if constexpr (BITS == 2) return 16 * (i >> 4) + 4 * (i & 3) + ((i & 15) >> 2);
    return i;
}
// in-place factor f_k of K position k
template <int BITS>
__device__ __forceinline__ int kfac_i8(int k)
{
    if constexpr (BITS == 4) return ((k >> 2) & 1) ? 16 : 1;
    if constexpr (BITS == 2) return 1 << (2 * ((k >> 2) & 3));
    return 1;
}

// K: one word of codes -> bytes f_k u (codes left in place)
template <int BITS>
__device__ __forceinline__ void k_bytes(uint32_t w, uint32_t* o)
{
    if constexpr (BITS == 4) {
        o[0] = w & 0x0F0F0F0Fu;
        o[1] = w & 0xF0F0F0F0u;
    } else if constexpr (BITS == 2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = w & (0x03030303u << (2 * j));
    } else {
        o[0] = w;
    }
}
// V: one word of codes -> bytes u
template <int BITS>
__device__ __forceinline__ void v_bytes(uint32_t w, uint32_t* o)
{
    if constexpr (BITS == 4) {
        o[0] = w & 0x0F0F0F0Fu;
        o[1] = (w >> 4) & 0x0F0F0F0Fu;
    } else if constexpr (BITS == 2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = (w >> (2 * j)) & 0x03030303u;
    } else {
        o[0] = w;
    }
}

// K row of one token (its chunks permuted by `sw`, see k_swizzle) -> bytes
// f_k u in tensor memory columns [0, 32) of this thread's lane.
template <int BITS>
__device__ __forceinline__ void k_row_to_tmem_u8(const uint8_t* row, uint32_t taddr, int sw)
{
    uint32_t o[16];
    auto chunk = [&](int c) { return *reinterpret_cast<const uint4*>(row + 16 * (c ^ sw)); };
    if constexpr (BITS == 4) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 a = chunk(2 * h);
            const uint4 b = chunk(2 * h + 1);
            k_bytes<4>(a.x, o); k_bytes<4>(a.y, o + 2); k_bytes<4>(a.z, o + 4); k_bytes<4>(a.w, o + 6);
            k_bytes<4>(b.x, o + 8); k_bytes<4>(b.y, o + 10); k_bytes<4>(b.z, o + 12); k_bytes<4>(b.w, o + 14);
            tmem_st16(taddr + 16 * h, o);
        }
    } else if constexpr (BITS == 2) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 a = chunk(h);
            k_bytes<2>(a.x, o); k_bytes<2>(a.y, o + 4); k_bytes<2>(a.z, o + 8); k_bytes<2>(a.w, o + 12);
            tmem_st16(taddr + 16 * h, o);
        }
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 a = chunk(4 * h + q);
                o[4 * q] = a.x; o[4 * q + 1] = a.y; o[4 * q + 2] = a.z; o[4 * q + 3] = a.w;
            }
            tmem_st16(taddr + 16 * h, o);
        }
    }
}

// V codes of dimension `dim` for the tile's 128 tokens -> 32 words of
// unsigned bytes in K-position order (registers; stored once the previous
// PV product has drained).  vblk0 and bb as for v_col_to_tmem.
template <int BITS, int Q0 = 0, int NQ = 4>
__device__ __forceinline__ void v_col_u8(const uint8_t* vblk0, int bb, int lp, int dim,
                                         uint32_t* o_all)
{
    const int P = 1 << lp;
    // 32 tokens per chunk: 16 bytes (4-bit), 8 bytes (2-bit), 32 bytes (8-bit);
    // chunks Q0 .. Q0 + NQ - 1 go to o_all[0 .. 8 NQ)
    const int row_bytes = P * BITS / 8;
    uint32_t* o = o_all - 8 * Q0;
#pragma unroll
    for (int q = Q0; q < Q0 + NQ; ++q) {
        const int t0 = 32 * q;
        const int pg = t0 >> lp, in = t0 & (P - 1);
        const uint8_t* row = vblk0 + pg * bb + dim * row_bytes;
        if constexpr (BITS == 4) {
            uint32_t w[4];
            if (P >= 32) {
                const uint4 x = *reinterpret_cast<const uint4*>(row + in / 2);
                w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
            } else {
                const uint2 x = *reinterpret_cast<const uint2*>(row);
                const uint2 y = *reinterpret_cast<const uint2*>(row + bb);
                w[0] = x.x; w[1] = x.y; w[2] = y.x; w[3] = y.y;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) v_bytes<4>(w[i], o + 8 * q + 2 * i);
        } else if constexpr (BITS == 2) {
            uint32_t w[2];
            if (P >= 32) {
                const uint2 x = *reinterpret_cast<const uint2*>(row + in / 4);
                w[0] = x.x; w[1] = x.y;
            } else {
                w[0] = *reinterpret_cast<const uint32_t*>(row);
                w[1] = *reinterpret_cast<const uint32_t*>(row + bb);
            }
            v_bytes<2>(w[0], o + 8 * q);
            v_bytes<2>(w[1], o + 8 * q + 4);
        } else {
            uint4 x, y;
            if (P >= 32) {
                x = *reinterpret_cast<const uint4*>(row + in);
                y = *reinterpret_cast<const uint4*>(row + in + 16);
            } else {
                x = *reinterpret_cast<const uint4*>(row);
                y = *reinterpret_cast<const uint4*>(row + bb);
            }
            o[8 * q + 0] = x.x; o[8 * q + 1] = x.y; o[8 * q + 2] = x.z; o[8 * q + 3] = x.w;
            o[8 * q + 4] = y.x; o[8 * q + 5] = y.y; o[8 * q + 6] = y.z; o[8 * q + 7] = y.w;
        }
    }
}

__device__ __forceinline__ void umma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// balanced signed byte digits of x (|x| < 2^30): x = sum_d 256^d dd[d]
__device__ __forceinline__ void digits4(int x, int* dd)
{
#pragma unroll
    for (int d = 0; d < 3; ++d) {
        dd[d] = (int)(int8_t)(x & 0xFF);
        x = (x - dd[d]) >> 8;
    }
    dd[3] = x;
}

// exact int32 -> fp32 for |v| < 2^22 on the FP32/integer pipes
__device__ __forceinline__ float small_int_to_float(uint32_t v)
{
    return __int_as_float((int)v + 0x4B400000) - 12582912.f;
}

template <int BITS, int RG>
__global__ void __launch_bounds__(kTcThreads, i8_ctas_per_sm(BITS, RG))
k_decode_i8(const TcArgs a)
{
    using F = I8Fmt<BITS>;
    constexpr int NS = 4 * RG;                       // S / O columns: 4r + digit
    constexpr uint32_t kColAK = 0, kColAV = 32, kColS = 64, kColO = 64 + NS;
    // kind::i8, s32 accumulate, M = 128, N = NS.  S: A u8, B s8 K-major.
    // O: A u8, B u8 MN-major.
    constexpr uint32_t kIdescS = (2u << 4) | (0u << 7) | (1u << 10) |
                                 ((uint32_t)(NS >> 3) << 17) | (8u << 24);
    constexpr uint32_t kIdescO = (2u << 4) | (0u << 7) | (0u << 10) | (1u << 16) |
                                 ((uint32_t)(NS >> 3) << 17) | (8u << 24);
    constexpr uint32_t kQRow = (NS / 8) * 128;      // bytes per 16-deep K chunk of q''
    constexpr uint32_t kPRow = (NS / 16) * 128;     // bytes per 8-deep K group of P''

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* bar_s = full + kStages;
    uint64_t* bar_o = bar_s + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + 64);
    int* s_flag = reinterpret_cast<int*>(smem + 68);
    float* s_red = reinterpret_cast<float*>(smem + 128);             // [4][16]
    unsigned* s_redv = reinterpret_cast<unsigned*>(smem + 384);      // [4]
    float* s_rowfac = reinterpret_cast<float*>(smem + 400);          // [16]
    float* s_l = reinterpret_cast<float*>(smem + 464);               // [4][16]
    int* s_init = reinterpret_cast<int*>(smem + 768);                // [NS] accumulator start
    int* s_pid = reinterpret_cast<int*>(smem + kI8Pid);
    unsigned long long* s_ps = reinterpret_cast<unsigned long long*>(smem + kI8Ps);
    uint8_t* s_qb = smem + kI8Hdr;                                   // q'' digits: 128 x NS bytes
    uint8_t* s_pb = s_qb + 128 * NS;                                 // P'' digits: 128 x NS bytes
    float* s_qf = reinterpret_cast<float*>(s_pb + 128 * NS);         // [RG][128] staging
    uint8_t* ring = reinterpret_cast<uint8_t*>(s_qf) + RG * 512;

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

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tok_begin = split * a.split_tokens;
    const int tok_end = min(seq_len, tok_begin + a.split_tokens);
    const int ntiles = (tok_end - tok_begin + kTile - 1) / kTile;
    const int P = a.page_size;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], kTcThreads / 32);
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        s_flag[0] = 0;
        fence_barrier_init();
    }
    __syncthreads();

    // bulk copies of a tile, shared by the 4 warps
    auto issue_tile = [&](uint8_t* stg, uint64_t* bar, const int* pids, int t0) {
        issue_tile_warps(stg, bar, a, pids, kvh, min(kTile, tok_end - t0), warp, lane);
    };
    for (int s = 0; s < kStages && s < ntiles; ++s) {
        const int t0 = tok_begin + s * kTile;
        issue_tile(ring + s * F::kStage, &full[s],
                   a.page_table + (int64_t)b * a.max_pages + (t0 >> a.lp), t0);
    }

    load_split_pids(s_pid, a, b, tok_begin, tok_end, tid);   // visible after the next barrier

    // ---- query rows: rotate, log2 scale, fixed point q'' with |q''| < 2^22
    for (int rr = warp; rr < RG; rr += 4) {
        const int r = rg * RG + rr;
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
        fwht128_lane(x, lane);
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[e] *= kLog2eTc / kHeadDim;
            amax = fmaxf(amax, fabsf(x[e]));
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, m));
        const int ex = amax > 0.f ? max(-100, ilogbf(amax)) : 0;
        const float pre = pow2i(21 - ex);           // largest |q''| in [2^21, 2^22)
#pragma unroll
        for (int e = 0; e < 4; ++e) s_qf[rr * kHeadDim + 4 * lane + e] = rintf(x[e] * pre);
        if (lane == 0) s_rowfac[rr] = pow2i(ex - 21) * (1.f / (float)F::F);
    }
    __syncthreads();
    {
        // K position k = tid holds dimension perm(k) with in-place factor f_k;
        // column 4 r + d holds digit d of (F / f_k) q''_r
        const int k = tid;
        const int dim = perm_i8<BITS>(k);
        const int fk = kfac_i8<BITS>(k);
        int dsum[NS];
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            int dd[4];
            digits4((int)s_qf[r * kHeadDim + dim] * (F::F / fk), dd);
#pragma unroll
            for (int d = 0; d < 4; ++d) {
                const int n = 4 * r + d;
                const int cm = (k >> 4) * (NS / 8) + (n >> 3);
                s_qb[cm * 128 + (n & 7) * 16 + (k & 15)] = (uint8_t)(int8_t)dd[d];
                dsum[n] = fk * dd[d];
            }
        }
        // accumulator start: -L sum_k f_k B[k][n], summed per warp by
        // shuffles, then over the 4 warps in the (idle) P'' buffer
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            int v = dsum[i];
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
            dsum[i] = v;
        }
        int* s_sum = reinterpret_cast<int*>(s_pb);                   // [4][NS]
        if (lane == 0)
#pragma unroll
            for (int i = 0; i < NS; ++i) s_sum[warp * NS + i] = dsum[i];
        __syncthreads();
        if (tid < NS) {
            int v = 0;
            for (int w = 0; w < 4; ++w) v += s_sum[w * NS + tid];
            s_init[tid] = -F::L * v;
        }
    }
    float rowfac[RG];
#pragma unroll
    for (int r = 0; r < RG; ++r) rowfac[r] = s_rowfac[r];
    fence_proxy_async_smem();
    // tensor memory last: a CTA resident beyond the 4 whose columns fit
    // waits here with its first tiles requested and its query operand staged
    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * warp) << 16);
    // accumulator start of S: registers for 4 rows, re-read from shared
    // memory for 8 (register pressure)
    constexpr int kInitRegs = RG <= 4 ? NS : 1;
    uint32_t sinit[kInitRegs];
#pragma unroll
    for (int n = 0; n < kInitRegs; ++n) sinit[n] = (uint32_t)s_init[n];
    const uint64_t desc_q = smem_desc(s_qb, kQRow, 128);
    const uint64_t desc_p = smem_desc(s_pb, kPRow, 128);

    float m_run[RG], l_run[RG], o_reg[RG];
    unsigned long long psum[RG];        // this thread's tokens: sum of P'' since the last fold
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        m_run[r] = -CUDART_INF_F;
        l_run[r] = 0.f;
        o_reg[r] = 0.f;
        psum[r] = 0ull;
    }
    int ev = 0;
    float vn = 1.f;
    float vlimit = __uint_as_float(1u << 23);
    const float kinv = 1.f / (float)F::L;
    const int lim_min = seq_len - a.q_len + (rg * RG) / a.group;
    const int kpos = perm_i8_inv<BITS>(tid);
    bool aborted = false;
    bool o_acc = false;                 // O holds an int32 sum to extend

    // per-warp sums of psum -> s_ps (the caller synchronises before folding)
    auto stash_psum = [&]() {
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            unsigned long long v = psum[r];
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
            if (lane == 0) s_ps[warp * 16 + r] = v;
        }
    };
    // fold O (sum u P'', int32 digits) minus L sum P'' into o_reg (dimension
    // tid); scale_now = 2^(ev - 127) 2^-22
    auto flush_o = [&](float scale_now) {
        uint32_t ov[NS];
#pragma unroll
        for (int c = 0; c < NS; c += 16) tmem_ld16(t_lane + kColO + c, ov + c);
        tmem_wait_ld();
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            const unsigned long long ps = s_ps[r] + s_ps[16 + r] + s_ps[32 + r] + s_ps[48 + r];
            // digit sums are non-negative and below 2^31
            const long long sum = (long long)ov[4 * r] + ((long long)ov[4 * r + 1] << 8) +
                                  ((long long)ov[4 * r + 2] << 16) + ((long long)ov[4 * r + 3] << 24);
            const long long v = sum - (long long)F::L * (long long)ps;
            o_reg[r] = fmaf((float)v, scale_now, o_reg[r]);
            psum[r] = 0ull;
        }
    };

    // Software pipeline: S = K q'' of tile t + 1 is issued as soon as its K
    // codes are in tensor memory, so it runs while tile t's softmax, V
    // staging and PV product proceed; PV(t) drains while tile t + 1's
    // scores are read and tile t + 2's K codes are staged.
    //
    // K codes of a tile -> A_K, accumulator start -> S, scales -> registers.
    auto stage_k = [&](int t, float& ks_out, float& vs_out) {
        const uint8_t* st = ring + (t % kStages) * F::kStage;
        const int pg = tid >> a.lp, row = tid & (P - 1);
        const uint8_t* kblk = st + pg * 2 * a.block_bytes;     // stage: [page][K block, V block]
        const uint8_t* vblk = kblk + a.block_bytes;
        k_row_to_tmem_u8<BITS>(kblk + row * F::CB, t_lane + kColAK, k_swizzle<BITS>(row));
        if constexpr (RG <= 4) {
            tmem_st16(t_lane + kColS, sinit);
        } else {
#pragma unroll
            for (int c = 0; c < NS; c += 16) {
                uint32_t iv[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint4 x = reinterpret_cast<const uint4*>(s_init + c)[q4];
                    iv[4 * q4] = x.x; iv[4 * q4 + 1] = x.y; iv[4 * q4 + 2] = x.z; iv[4 * q4 + 3] = x.w;
                }
                tmem_st16(t_lane + kColS + c, iv);
            }
        }
        ks_out = reinterpret_cast<const float*>(kblk + P * F::CB)[row] * kinv;
        vs_out = reinterpret_cast<const float*>(vblk + P * F::CB)[row] * kinv;
        if (tok_begin + t * kTile + tid >= tok_end) { ks_out = 0.f; vs_out = 0.f; }
    };
    // One thread issues the 4 K-steps of a product and commits them: MMAs
    // accumulating into one tensor-memory accumulator stay in one thread's
    // issue order (S from thread 0, O from thread 96).
    auto issue_qk = [&]() {
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 4; ++j)
            umma_i8_ts(tmem + kColS, tmem + kColAK + 8 * j, desc_q + ((2 * j * kQRow) >> 4), kIdescS,
                       1u);
        umma_commit(bar_s);
    };
    auto issue_pv = [&]() {
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < 4; ++j)
            umma_i8_ts(tmem + kColO, tmem + kColAV + 8 * j, desc_p + ((4 * j * kPRow) >> 4),
                       kIdescO, 1u);
        umma_commit(bar_o);
    };
    // O starts (and restarts after each fold) at zero: every PV step accumulates
    auto zero_o = [&]() {
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
        for (int c = 0; c < NS; c += 16) tmem_st16(t_lane + kColO + c, z);
    };

    float ks, vs;                       // scales of the tile whose scores come next
    {
        bool ok = mbar_wait_sleep(&full[0], 0u, kPollsTc);
        tc_fence_after();
        if (!ok) atomicOr(&s_flag[0], 1);
        stage_k(0, ks, vs);
        zero_o();
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (s_flag[0]) aborted = true;
        else if (tid == 0) issue_qk();
    }

    for (int tt = 0; tt < ntiles && !aborted; ++tt) {
        const int stage = tt % kStages;
        uint8_t* st = ring + stage * F::kStage;
        const int tok0 = tok_begin + tt * kTile;
        const int tok = tok0 + tid;

        // a. scores of tile tt
        bool ok = mbar_wait_sleep(bar_s, (uint32_t)(tt & 1), kPollsTc);
        tc_fence_after();
        uint32_t sraw[NS];
#pragma unroll
        for (int c = 0; c < NS; c += 16) tmem_ld16(t_lane + kColS + c, sraw + c);

        // b. V column of dimension tid (registers), overlapping the load of
        // S for 4 rows; after the scores for 8 (register pressure)
        uint32_t vw[32];
        if constexpr (RG <= 4) v_col_u8<BITS>(st + a.block_bytes, 2 * a.block_bytes, a.lp, tid, vw);
        tmem_wait_ld();

        const bool full_tile = tok0 + kTile - 1 <= lim_min;
        float sc[RG];
        bool need = false;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            float v = small_int_to_float(sraw[4 * r + 1]) * 256.f + small_int_to_float(sraw[4 * r]);
            v = fmaf(small_int_to_float(sraw[4 * r + 2]), 65536.f, v);
            if constexpr (BITS != 8) v = fmaf(small_int_to_float(sraw[4 * r + 3]), 16777216.f, v);
            float x = v * (ks * rowfac[r]);
            if (!full_tile) {
                const int R = rg * RG + r;
                const int lr = R < a.G ? seq_len - a.q_len + R / a.group : -1;
                x = tok <= lr ? x : -CUDART_INF_F;
            }
            sc[r] = x;
            need |= x > m_run[r] + kLazyTc;
        }
        need |= vs >= vlimit;
        const float vs_t = vs;
        if constexpr (RG > 4) v_col_u8<BITS>(st + a.block_bytes, 2 * a.block_bytes, a.lp, tid, vw);

        // c. K codes of tile tt + 1 (S of tile tt is in registers)
        if (tt + 1 < ntiles) {
            ok = ok && mbar_wait_sleep(&full[(tt + 1) % kStages], (uint32_t)(((tt + 1) / kStages) & 1),
                                       kPollsTc);
            tc_fence_after();
            stage_k(tt + 1, ks, vs);
        }

        // d. PV(tt - 1) has drained: A_V, O and the P'' buffer are free
        if (tt > 0) {
            ok = ok && mbar_wait_sleep(bar_o, (uint32_t)((tt - 1) & 1), kPollsTc);
            tc_fence_after();
        }
        if (!ok) atomicOr(&s_flag[0], 1);
        tmem_st16(t_lane + kColAV, vw);
        tmem_st16(t_lane + kColAV + 16, vw + 16);
        tmem_wait_st();
        tc_fence_before();

        // e. one barrier: tile tt + 1's operands are staged, stage tt is consumed
        const int any = __syncthreads_or(need);
        if (s_flag[0]) { aborted = true; break; }
        if (tid == 0 && tt + 1 < ntiles) issue_qk();
        if (tt + kStages < ntiles) {
            const int t0 = tok_begin + (tt + kStages) * kTile;
            issue_tile(st, &full[stage], s_pid + ((t0 - tok_begin) >> a.lp), t0);
        }

        // f. rare: new row maxima or a larger V scale exponent
        if (any) {
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                float v = sc[r];
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
                if (lane == 0) s_red[warp * 16 + r] = v;
            }
            const unsigned vb = __reduce_max_sync(kFull, __float_as_uint(vs_t));
            if (lane == 0) s_redv[warp] = vb;
            if (o_acc) stash_psum();
            __syncthreads();
            if (o_acc) {
                flush_o(pow2i(ev - 127 - 22));
                zero_o();
                tmem_wait_st();
            }
            o_acc = false;
            const unsigned vmax = max(max(s_redv[0], s_redv[1]), max(s_redv[2], s_redv[3]));
            ev = max(ev, (int)(vmax >> 23));
            vn = pow2i(127 - ev);
            vlimit = ev >= 254 ? CUDART_INF_F : __uint_as_float((uint32_t)(ev + 1) << 23);
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                const float tmax = fmaxf(fmaxf(s_red[r], s_red[16 + r]),
                                         fmaxf(s_red[32 + r], s_red[48 + r]));
                const float mn = fmaxf(m_run[r], tmax);
                const float alpha = mn == -CUDART_INF_F ? 1.f : fast_exp2(m_run[r] - mn);
                m_run[r] = mn;
                l_run[r] *= alpha;
                o_reg[r] *= alpha;
            }
            tc_fence_before();
            __syncthreads();
        }

        // g. P'' row of token tid at K position kpos: 4 digit bytes per row
        const float vn_t = vs_t * vn * 4194304.f;       // 2^22 fixed point
        uint32_t pw[RG];
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            float pr = fast_exp2(sc[r] - m_run[r]);
            if (!full_tile) pr = sc[r] == -CUDART_INF_F ? 0.f : pr;
            l_run[r] += pr;
            pw[r] = pr > 0.f ? __float2uint_rn(pr * vn_t) : 0u;
            psum[r] += pw[r];
        }
        {
            uint8_t* rowp = s_pb + (kpos >> 3) * kPRow + (kpos & 7) * 16;
#pragma unroll
            for (int ng = 0; ng < RG / 4; ++ng)
                *reinterpret_cast<uint4*>(rowp + ng * 128) =
                    make_uint4(pw[4 * ng], pw[4 * ng + 1], pw[4 * ng + 2], pw[4 * ng + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // h. O^T += V^T P'' (warp 3, which issued the fewest copies)
        if (tid == 96) issue_pv();
        o_acc = true;
    }

    // ---- epilogue
    bool ok = !aborted && mbar_wait_sleep(bar_o, (uint32_t)((ntiles - 1) & 1), kPollsTc);
    tc_fence_after();
    ok = __syncthreads_and(ok);
    const int nrows = min(RG, a.G - rg * RG);
    float* sO = reinterpret_cast<float*>(ring);          // [RG][128]
    if (ok) {
        stash_psum();
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            float l = l_run[r];
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) l += __shfl_xor_sync(kFull, l, m);
            if (lane == 0) s_l[warp * 16 + r] = l;
        }
        __syncthreads();
        if (o_acc) flush_o(pow2i(ev - 127 - 22));
#pragma unroll
        for (int r = 0; r < RG; ++r) sO[r * kHeadDim + tid] = o_reg[r];
    } else if (tid == 0) {
        report_error(a.err, TQ_ERR_TIMEOUT, kErrWaitTile);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    tc_finish<RG, 16>(a, sO, s_l, m_run, s_flag, b, kvh, rg, split, nsplit, nrows, warp, lane, tid,
                  ok, (int64_t)b * gridDim.y + blockIdx.y);
}

template <int BITS, int RG, bool FP8 = false>
cudaError_t launch_tc(const TcArgs& a, dim3 grid, cudaStream_t stream)
{
    constexpr int NCOL = 2 * RG < 16 ? 16 : 2 * RG;
    const size_t smem = TcHdr<RG>::kBytes + 2 * 256 * NCOL + (size_t)kStages * TcFmt<BITS, FP8>::kStage;
    static int configured = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 31 || !(configured & (1 << dev))) {
        e = cudaFuncSetAttribute(k_decode_tc<BITS, RG, FP8>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 31) configured |= 1 << dev;
    }
    k_decode_tc<BITS, RG, FP8><<<grid, kTcThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int BITS, int RG>
cudaError_t launch_i8(const TcArgs& a, dim3 grid, cudaStream_t stream)
{
    constexpr int NS = 4 * RG;
    const size_t smem = kI8Hdr + 2 * 128 * NS + RG * 512 + (size_t)kStages * I8Fmt<BITS>::kStage;
    static int configured = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 31 || !(configured & (1 << dev))) {
        e = cudaFuncSetAttribute(k_decode_i8<BITS, RG>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 31) configured |= 1 << dev;
    }
    k_decode_i8<BITS, RG><<<grid, kTcThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

// ===================================================================
// Query-major kernel for long verify windows and prefill chunks (turbo
// formats, G = q_len x GQA >= 128 rows per kv head).
//
// One CTA (256 threads) owns 128 query rows of one (sequence, kv head) and
// walks every key tile its rows may see (causal), so each K/V tile is
// dequantised once for 128 rows instead of once per 16-row group:
//   1. thread t < 128 unpacks token t's K row, thread 128 + d dimension d's V
//      column, into exact f16 integers in shared memory, in the canonical
//      K-major layout (8x8 core matrices) of the MMA's B operand; the tile's
//      K and V scales go to shared memory too.
//   2. one thread issues S[128 rows][128 keys] = Q' K^T: A = Q' in tensor
//      memory (the rotated query, prescaled per row, split into f16 hi and
//      lo parts: two MMA chains into one fp32 accumulator).
//   3. two threads own row r (warps w and w + 4 reach the same tensor-memory
//      lanes), one per half of the keys: each reads its scores (twice: the
//      row maximum, exchanged through shared memory, then the weights),
//      scales them by s_k / L and the row factor, masks keys beyond the
//      row's causal limit, and runs an online softmax with a lazy maximum (a
//      warp rescales its half of its rows of O only when one of them gains
//      more than 2^8).  P' = p s_v / L 2^(127 - ev), split hi/lo in f16, goes
//      to tensor memory as the A operand of the PV product (keys in the V
//      unpacker's pair order).
//   4. one thread issues O[128 rows][128 dims] += P' V (two chains).
// The epilogue normalises each row, rotates it back (a 128-point FWHT in
// the thread's registers) and writes it; there is no split merge.
// Tensor memory: Q' hi/lo 128 columns, S 128, O 128, P' hi/lo 128.
// ===================================================================
constexpr int kPfRows = 128;
constexpr int kPfThreads = 256;
constexpr uint32_t kPfColQ = 0, kPfColS = 128, kPfColO = 256, kPfColP = 384;
constexpr uint32_t kPfTmemCols = 512;
// shared memory (bytes from the start)
constexpr int kPfKs = 128;          // [128] K scales of the tile, / L
constexpr int kPfVs = 640;          // [128] V scales of the tile, / L
constexpr int kPfRowfac = 1152;     // [128] row factors
constexpr int kPfPmax = 1664;       // [2][128] row maxima of the two key halves
constexpr int kPfL = 2688;          // [2][128] row sums of the two key halves
constexpr int kPfKdeq = 4096;       // [128 keys x 128 dims] f16, B of S
constexpr int kPfVdeq = kPfKdeq + 32768;   // [2][128 dims x 128 keys] f16, B of O, by tile parity
constexpr int kPfRing = kPfVdeq + 2 * 32768;   // [kStages] tile stages

// K-major core-matrix offset (bytes) of element (n, k) of a [128 x 128] f16
// B operand: 8x8 core matrices of 128 bytes, N-adjacent ones 128 bytes
// apart, K-adjacent ones 16 x 128 bytes apart.
__device__ __forceinline__ int pf_b_offset(int n, int k)
{
    return ((k >> 3) * 16 + (n >> 3)) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

template <int BITS>
__global__ void __launch_bounds__(kPfThreads, 1)
k_prefill_tc(const TcArgs a)
{
    using F = TcFmt<BITS>;
    // f32 accumulate, f16 A (tensor memory) and B (shared, K-major), M = 128, N = 128
    constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(128 >> 3) << 17) | (8u << 24);
    constexpr uint32_t kLbo = 16 * 128;             // K-adjacent core matrices

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);              // [kStages]
    uint64_t* bar_s = full + kStages;
    uint64_t* bar_o = bar_s + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + 64);
    int* s_flag = reinterpret_cast<int*>(smem + 68);
    float* s_ks = reinterpret_cast<float*>(smem + kPfKs);
    float* s_vs = reinterpret_cast<float*>(smem + kPfVs);
    float* s_rowfac = reinterpret_cast<float*>(smem + kPfRowfac);
    float* s_pmax = reinterpret_cast<float*>(smem + kPfPmax);
    float* s_lsum = reinterpret_cast<float*>(smem + kPfL);
    uint8_t* kdeq = smem + kPfKdeq;
    uint8_t* vdeq0 = smem + kPfVdeq;
    uint8_t* ring = smem + kPfRing;

    const int rb = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int seq_len = a.seq_lens[b];
    if (seq_len < a.q_len || seq_len > a.max_seq_len) {
        if (rb == 0 && kvh == 0 && tid == 0) report_error(a.err, TQ_ERR_DEVICE_CHECK, kErrSeqLen);
        return;
    }
    const int P = a.page_size;
    // this thread's row (tensor-memory lane) and half of the keys; the row's
    // causal limit; the block's last visible key
    const int r = 32 * (warp & 3) + lane, hk = warp >> 2;
    const int R = rb * kPfRows + r;
    const bool row_ok = R < a.G;
    const int tq = row_ok ? R / a.group : 0;
    const int h = kvh * a.group + (R - tq * a.group);
    const int lim = row_ok ? seq_len - a.q_len + tq : -1;
    const int r_last = min(a.G, (rb + 1) * kPfRows) - 1;
    const int nkeys = seq_len - a.q_len + r_last / a.group + 1;     // <= seq_len
    const int ntiles = (nkeys + kTile - 1) / kTile;
    const int32_t* pt = a.page_table + (int64_t)b * a.max_pages;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        s_flag[0] = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, kPfTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t t_lane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);

    if (warp == 0)
        for (int s = 0; s < kStages && s < ntiles; ++s)
            issue_tile_tc(ring + s * F::kStage, &full[s], a, pt + ((s * kTile) >> a.lp), kvh,
                          min(kTile, nkeys - s * kTile), lane);

    // ---- Q' of this row (first half of the threads): rotate (128-point
    // FWHT in registers), log2 scale, power-of-two prescale, f16 hi + lo in
    // the K unpacker's dimension order
    if (hk == 0) {
        float x[kHeadDim];
        if (row_ok) {
            const uint4* src = reinterpret_cast<const uint4*>(
                a.q + (((int64_t)b * a.q_len + tq) * a.num_q_heads + h) * kHeadDim);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 w = __ldg(src + c);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * c + 2 * e] = bf16_bits_to_float(ww[e] & 0xffffu);
                    x[8 * c + 2 * e + 1] = bf16_bits_to_float(ww[e] >> 16);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < kHeadDim; ++i) x[i] = 0.f;
        }
#pragma unroll
        for (int hs = 1; hs < kHeadDim; hs <<= 1)
#pragma unroll
            for (int i = 0; i < kHeadDim; ++i)
                if (!(i & hs)) {
                    const float u = x[i], v = x[i + hs];
                    x[i] = u + v;
                    x[i + hs] = u - v;
                }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < kHeadDim; ++i) {
            x[i] *= kLog2eTc / kHeadDim;        // (H q / sqrt d) . y / sqrt d = (H q) . y / d
            amax = fmaxf(amax, fabsf(x[i]));
        }
        const int ex = amax > 0.f ? max(-100, min(100, ilogbf(amax))) : 0;
        const float pre = pow2i(12 - ex);
        s_rowfac[r] = pow2i(ex - 12);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t hw[16], lw[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
                const int k0 = 32 * c + 2 * w;
                const float q0 = x[perm_k<F::GB>(k0)] * pre, q1 = x[perm_k<F::GB>(k0 + 1)] * pre;
                hw[w] = split_hi_lo<true>(q0, q1, true);
                lw[w] = split_hi_lo<true>(q0, q1, false);
            }
            tmem_st16(t_lane + kPfColQ + 16 * c, hw);
            tmem_st16(t_lane + kPfColQ + 64 + 16 * c, lw);
        }
        tmem_wait_st();                           // complete before the first S product
    }

    __syncthreads();                              // row factors
    const float rowfac = s_rowfac[r];
    const uint64_t desc_k = smem_desc(kdeq, kLbo, 128);
    const uint64_t desc_v0 = smem_desc(vdeq0, kLbo, 128);
    const float kinv = F::kDequant;
    float m_run = -CUDART_INF_F, l_run = 0.f;
    int ev = 0;                                   // running V-scale exponent (biased), CTA-uniform
    float vn = 1.f;                               // 2^(127 - ev)
    bool aborted = false;

    for (int t = 0; t < ntiles; ++t) {
        const int stage = t % kStages;
        uint8_t* st = ring + stage * F::kStage;
        const int tok0 = t * kTile;
        uint8_t* vdeq = vdeq0 + (t & 1) * 32768;
        // the V buffer of this tile was last read by PV(t - 2), which drained
        // before tile t - 1's weights were written
        bool ok = mbar_wait_sleep(&full[stage], (uint32_t)((t / kStages) & 1), kPollsTc);
        tc_fence_after();
        if (!ok) atomicOr(&s_flag[0], 1);

        // 1. token u's K row (threads u < 128) or dimension u's V column
        // (threads 128 + u) -> f16 B operands; token u's K or V scale
        {
            const int u = tid & (kTile - 1);
            const int pg = u >> a.lp, row = u & (P - 1);
            const uint8_t* kblk = st + pg * 2 * a.block_bytes;
            const uint8_t* vblk = kblk + a.block_bytes;
            const bool live = tok0 + u < nkeys;
            if (hk == 0) {
                k_row_unpack<BITS>(kblk + row * F::CB, k_swizzle<BITS>(row),
                                   [&](int c, const uint32_t* o) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4*>(kdeq + pf_b_offset(u, 2 * (c + 4 * i))) =
                            make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                });
                s_ks[u] = live ? reinterpret_cast<const float*>(kblk + P * F::CB)[row] * kinv : 0.f;
            } else {
                v_col_unpack<BITS>(st + a.block_bytes, 2 * a.block_bytes, a.lp, u,
                                   [&](int c, const uint32_t* o) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4*>(vdeq + pf_b_offset(u, 2 * (c + 4 * i))) =
                            make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                });
                s_vs[u] = live ? reinterpret_cast<const float*>(vblk + P * F::CB)[row] * kinv : 0.f;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();                          // also: the stage is consumed
        if (s_flag[0]) { aborted = true; break; }
        if (warp == 0 && t + kStages < ntiles)
            issue_tile_tc(st, &full[stage], a, pt + (((t + kStages) * kTile) >> a.lp), kvh,
                          min(kTile, nkeys - (t + kStages) * kTile), lane);

        // 2. S = Q' K^T (hi, then lo)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                umma_f16_ts(tmem + kPfColS, tmem + kPfColQ + 8 * j, desc_k + ((2 * j * kLbo) >> 4),
                            kIdesc, j > 0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                umma_f16_ts(tmem + kPfColS, tmem + kPfColQ + 64 + 8 * j,
                            desc_k + ((2 * j * kLbo) >> 4), kIdesc, 1u);
            umma_commit(bar_s);
        }

        // the tile's largest V scale (every thread reads all of them: uniform)
        unsigned vmaxb = 0;
#pragma unroll 8
        for (int i = 0; i < kTile; i += 4) {
            const uint4 x = *reinterpret_cast<const uint4*>(s_vs + i);
            vmaxb = max(max(vmaxb, max(x.x, x.y)), max(x.z, x.w));
        }
        const int ev_new = max(ev, (int)(vmaxb >> 23));

        ok = mbar_wait_sleep(bar_s, (uint32_t)(t & 1), kPollsTc);
        tc_fence_after();
        if (!ok) atomicOr(&s_flag[0], 1);

        // 3a. this row's maximum over the tile: each thread its half of the
        // keys (the row factor is a positive constant: applied after)
        float hmax = -CUDART_INF_F;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * hk + cc;
            uint32_t v[32];
            tmem_ld16(t_lane + kPfColS + 32 * c, v);
            tmem_ld16(t_lane + kPfColS + 32 * c + 16, v + 16);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 ks4 = *reinterpret_cast<const float4*>(s_ks + 32 * c + i);
                const float kk[4] = {ks4.x, ks4.y, ks4.z, ks4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = 32 * c + i + e;
                    const float xs = __uint_as_float(v[i + e]) * kk[e];
                    hmax = fmaxf(hmax, tok0 + key <= lim ? xs : -CUDART_INF_F);
                }
            }
        }
        s_pmax[hk * kPfRows + r] = hmax;
        // PV(t - 1) has drained (it ran under this tile's unpack, S product
        // and maximum): O and the P' columns are free
        if (t > 0) {
            ok = mbar_wait_sleep(bar_o, (uint32_t)((t - 1) & 1), kPollsTc);
            tc_fence_after();
            if (!ok) atomicOr(&s_flag[0], 1);
        }
        __syncthreads();
        const float sfac = rowfac;
        const float tmax = fmaxf(s_pmax[r], s_pmax[kPfRows + r]) * sfac;
        // rescale O (this warp's rows) when a row gains more than 2^8 or the
        // V-scale exponent grows
        const float mn = fmaxf(m_run, tmax);
        const bool grow = mn > m_run + kLazyTc;
        const float m_use = grow ? mn : m_run;
        const float alpha = (grow && m_run != -CUDART_INF_F) ? fast_exp2(m_run - mn) : 1.f;
        const float av = pow2i(ev - ev_new);
        if (t > 0 && (__any_sync(kFull, alpha != 1.f) || ev_new != ev)) {
            const float f = alpha * av;
#pragma unroll
            for (int c = 64 * hk; c < 64 * hk + 64; c += 16) {
                uint32_t ov[16];
                tmem_ld16(t_lane + kPfColO + c, ov);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
                tmem_st16(t_lane + kPfColO + c, ov);
            }
        }
        l_run *= alpha;
        m_run = m_use;
        ev = ev_new;
        vn = pow2i(127 - ev);

        // 3b. weights of this row's half of the keys -> P' (hi, lo), keys in
        // the V unpacker's order
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * hk + cc;
            uint32_t v[32];
            tmem_ld16(t_lane + kPfColS + 32 * c, v);
            tmem_ld16(t_lane + kPfColS + 32 * c + 16, v + 16);
            tmem_wait_ld();
            float pv[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 ks4 = *reinterpret_cast<const float4*>(s_ks + 32 * c + i);
                const float4 vs4 = *reinterpret_cast<const float4*>(s_vs + 32 * c + i);
                const float kk[4] = {ks4.x, ks4.y, ks4.z, ks4.w};
                const float vv[4] = {vs4.x, vs4.y, vs4.z, vs4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = 32 * c + i + e;
                    const float xs = __uint_as_float(v[i + e]) * (kk[e] * sfac);
                    const float p = tok0 + key <= lim ? fast_exp2(xs - m_run) : 0.f;
                    l_run += p;
                    pv[i + e] = p * (vv[e] * vn);
                }
            }
            uint32_t hw[16], lw[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
                const float p0 = pv[perm_k<F::GB>(2 * w)], p1 = pv[perm_k<F::GB>(2 * w + 1)];
                hw[w] = split_hi_lo<true>(p0, p1, true);
                lw[w] = split_hi_lo<true>(p0, p1, false);
            }
            tmem_st16(t_lane + kPfColP + 16 * c, hw);
            tmem_st16(t_lane + kPfColP + 64 + 16 * c, lw);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();

        // 4. O += P' V (hi, then lo)
        if (tid == 0) {
            tc_fence_after();
            const uint64_t desc_v = desc_v0 + (uint64_t)(((t & 1) * 32768) >> 4);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                umma_f16_ts(tmem + kPfColO, tmem + kPfColP + 8 * j, desc_v + ((2 * j * kLbo) >> 4),
                            kIdesc, (t > 0 || j > 0) ? 1u : 0u);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                umma_f16_ts(tmem + kPfColO, tmem + kPfColP + 64 + 8 * j,
                            desc_v + ((2 * j * kLbo) >> 4), kIdesc, 1u);
            umma_commit(bar_o);
        }
    }

    // ---- epilogue (first half of the threads): normalise, rotate back,
    // write this row
    bool ok = !aborted && ntiles > 0 &&
              mbar_wait_sleep(bar_o, (uint32_t)((ntiles - 1) & 1), kPollsTc);
    tc_fence_after();
    s_lsum[hk * kPfRows + r] = l_run;
    ok = __syncthreads_and(ok);
    if (ok && hk == 0) {
        l_run = s_lsum[r] + s_lsum[kPfRows + r];
        float x[kHeadDim];
#pragma unroll
        for (int c = 0; c < kHeadDim; c += 16) {
            uint32_t ov[16];
            tmem_ld16(t_lane + kPfColO + c, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) x[c + i] = __uint_as_float(ov[i]);
        }
        const float inv = (l_run > 0.f ? 1.f / l_run : 0.f) * pow2i(ev - 127) *
                          0.08838834764831845f;     // V-scale exponent back, 1 / sqrt d
#pragma unroll
        for (int hs = 1; hs < kHeadDim; hs <<= 1)
#pragma unroll
            for (int i = 0; i < kHeadDim; ++i)
                if (!(i & hs)) {
                    const float u = x[i], v = x[i + hs];
                    x[i] = u + v;
                    x[i + hs] = u - v;
                }
        if (row_ok) {
            float4* dst = reinterpret_cast<float4*>(
                a.out + (((int64_t)b * a.q_len + tq) * a.num_q_heads + h) * kHeadDim);
#pragma unroll
            for (int c = 0; c < kHeadDim / 4; ++c)
                dst[c] = make_float4(x[4 * c] * inv, x[4 * c + 1] * inv, x[4 * c + 2] * inv,
                                     x[4 * c + 3] * inv);
        }
    } else if (tid == 0 && ntiles > 0) {
        report_error(a.err, TQ_ERR_TIMEOUT, kErrWaitTile);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kPfTmemCols);
    }
}

template <int BITS>
cudaError_t launch_prefill(const TcArgs& a, int batch, cudaStream_t stream)
{
    const size_t smem = kPfRing + (size_t)kStages * TcFmt<BITS>::kStage;
    static int configured = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 31 || !(configured & (1 << dev))) {
        e = cudaFuncSetAttribute(k_prefill_tc<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 31) configured |= 1 << dev;
    }
    const dim3 grid((unsigned)((a.G + kPfRows - 1) / kPfRows), (unsigned)a.num_kv_heads,
                    (unsigned)batch);
    k_prefill_tc<BITS><<<grid, kPfThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

// Query rows of one tensor-core CTA: 4, 8 or 16.  Up to 4 rows, 2-, 4- and
// 8-bit codes go to the integer kernel; 3-bit and fp8 codes, and every format
// with more than 4 rows per kv head, to the f16 kernel (its two columns per
// row, against the integer kernel's four digit columns, make it the faster
// one at 8 rows; 16 rows in one CTA read the kv head's pages once).
int decode_tc_rows(int format, int G)
{
    (void)format;
    return G <= 4 ? 4 : (G <= 8 ? 8 : 16);
}

// The query-major kernel takes 128 or more rows per kv head of a turbo format;
// it writes its rows directly (no splits, no workspace).
bool decode_uses_prefill(int format, int G)
{
    return format != TQ_FP8 && format != 16 && G >= kPfRows;
}

cudaError_t launch_decode_tc(const void* q, const tq_cache& c, int64_t block_bytes,
                             const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                             int batch, int q_len, int num_q_heads, int max_seq_len, float* out,
                             void* workspace, int split_tokens, cudaStream_t stream)
{
    TcArgs a{};
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
    a.page_size = c.page_size;
    a.lp = c.page_size == 16 ? 4 : (c.page_size == 32 ? 5 : 6);
    a.max_seq_len = max_seq_len;
    // 128 or more rows per kv head (prefill chunks, long verify windows),
    // turbo formats: the query-major kernel, one CTA per 128 rows
    if (decode_uses_prefill(c.format, a.G)) {
        switch (c.format) {
        case 2: return launch_prefill<2>(a, batch, stream);
        case 3: return launch_prefill<3>(a, batch, stream);
        case 4: return launch_prefill<4>(a, batch, stream);
        case 8: return launch_prefill<8>(a, batch, stream);
        default: return cudaErrorInvalidValue;
        }
    }
    const int rows = decode_tc_rows(c.format, a.G);
    a.R = (a.G + rows - 1) / rows;
    a.page_size = c.page_size;
    a.lp = c.page_size == 16 ? 4 : (c.page_size == 32 ? 5 : 6);
    a.split_tokens = split_tokens;
    a.max_splits = (max_seq_len + split_tokens - 1) / split_tokens;
    a.max_seq_len = max_seq_len;
    if (a.max_splits > 1) {
        const int64_t units = (int64_t)batch * c.num_kv_heads * a.R;
        const int64_t cnt = ((units * 4 + 255) / 256) * 256;
        const int64_t ml = ((units * a.max_splits * rows * 8 + 255) / 256) * 256;
        uint8_t* w = static_cast<uint8_t*>(workspace);
        a.ws_cnt = reinterpret_cast<uint32_t*>(w);
        a.ws_ml = reinterpret_cast<float2*>(w + cnt);
        a.ws_o = reinterpret_cast<float*>(w + cnt + ml);
    }
    const dim3 grid((unsigned)a.max_splits, (unsigned)(c.num_kv_heads * a.R), (unsigned)batch);
#define TQ_I8(B)                                                                    \
    return rows == 4   ? launch_i8<B, 4>(a, grid, stream)                              \
           : rows == 8 ? launch_tc<B, 8>(a, grid, stream)                              \
                       : launch_tc<B, 16>(a, grid, stream)
    switch (c.format) {
    case 2: TQ_I8(2);
    case 3:
        return rows == 4   ? launch_tc<3, 4>(a, grid, stream)
               : rows == 8 ? launch_tc<3, 8>(a, grid, stream)
                           : launch_tc<3, 16>(a, grid, stream);
    case 4: TQ_I8(4);
    case 8: TQ_I8(8);
    case TQ_FP8:
        return rows == 4   ? launch_tc<8, 4, true>(a, grid, stream)
               : rows == 8 ? launch_tc<8, 8, true>(a, grid, stream)
                           : launch_tc<8, 16, true>(a, grid, stream);
    default: return cudaErrorInvalidValue;
    }
#undef TQ_I8
}

}  // namespace tq
