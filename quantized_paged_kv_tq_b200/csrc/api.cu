// C ABI of libtq.so: argument checks on the host, then one kernel launch.
// The contract of every entry point is stated in include/tq.h.
#include <chrono>
#include <cstdint>
#include <new>
#include <thread>

#include <cuda_runtime.h>

#include "../../include/tq.h"

#define TQ_API extern "C" __attribute__((visibility("default")))

namespace tq {
cudaError_t launch_quantize_append(const void* k, const void* v, const int64_t* slots,
                                   int num_tokens, int bits, const tq_cache& c,
                                   int64_t block_bytes, cudaStream_t stream);
cudaError_t launch_append_bf16(const void* k, const void* v, const int64_t* slots,
                               int num_tokens, const tq_cache& c, cudaStream_t stream);
int decode_split_tokens(int page_size);
int decode_row_groups(int format, int G);
size_t decode_workspace_bytes(int batch, int num_kv_heads, int G, int max_seq_len,
                              int page_size, int format);
cudaError_t launch_decode(const void* q, const tq_cache& c, int64_t block_bytes,
                          const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                          int batch, int q_len, int num_q_heads, int max_seq_len, float* out,
                          void* workspace, cudaStream_t stream);
cudaError_t launch_hbm_copy(const void* src, void* dst, size_t bytes, cudaStream_t stream);
cudaError_t launch_hbm_read(const void* src, size_t bytes, uint32_t* sink, cudaStream_t stream);
}  // namespace tq

namespace {

constexpr int kMaxRows = 4096;        // q_len * GQA group: a verify window or a prefill chunk

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int format_bits(int32_t f)
{
    switch (f) {
    case TQ_TURBO2: return 2;
    case TQ_TURBO3: return 3;
    case TQ_TURBO4: return 4;
    case TQ_TURBO8: return 8;
    case TQ_FP8: return 8;
    case TQ_BF16: return 16;
    default: return 0;
    }
}

int64_t block_bytes(int32_t format, int32_t head_dim, int32_t page_size)
{
    const int b = format_bits(format);
    if (b == 0 || head_dim != 128) return 0;
    if (page_size != 16 && page_size != 32 && page_size != 64) return 0;
    if (b == 16) return (int64_t)page_size * head_dim * 2;
    return (int64_t)page_size * (head_dim * b / 8 + 4);
}

// Checks shared by every call that takes a cache descriptor.
tq_status check_cache(const tq_cache* c, bool want_turbo)
{
    if (!c) return TQ_ERR_INVALID_ARG;
    const int b = format_bits(c->format);
    if (b == 0) return TQ_ERR_INVALID_ARG;
    if (want_turbo != (b != 16)) return TQ_ERR_INVALID_ARG;
    if (c->head_dim <= 0 || c->page_size <= 0 || c->num_kv_heads <= 0 || c->num_pages <= 0)
        return TQ_ERR_INVALID_ARG;
    if (c->head_dim != 128) return TQ_ERR_UNSUPPORTED;
    if (c->page_size != 16 && c->page_size != 32 && c->page_size != 64) return TQ_ERR_UNSUPPORTED;
    if (!c->pages || !aligned16(c->pages)) return TQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(c->dev_error) & 3u) != 0) return TQ_ERR_INVALID_ARG;
    return TQ_OK;
}

tq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

tq_status check_append(const void* k, const void* v, const int64_t* slots, int32_t num_tokens,
                       const tq_cache* c, bool turbo)
{
    tq_status s = check_cache(c, turbo);
    if (s != TQ_OK) return s;
    if (num_tokens < 0) return TQ_ERR_INVALID_ARG;
    if (num_tokens == 0) return TQ_OK;
    if (!k || !v || !slots) return TQ_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(slots) & 7u))
        return TQ_ERR_INVALID_ARG;
    return TQ_OK;
}

}  // namespace

namespace tq {

// Host checks of a decode call except its workspace, shared by every decode
// entry point (tq_paged_decode, tq_paged_decode_bf16 and the no-alloc decode).
tq_status check_decode_call(const void* q, const tq_cache* c, const int32_t* page_table,
                            int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                            int32_t q_len, int32_t num_q_heads, int32_t max_seq_len,
                            const float* out, bool turbo)
{
    tq_status s = check_cache(c, turbo);
    if (s != TQ_OK) return s;
    if (batch < 0 || q_len <= 0 || num_q_heads <= 0 || max_seq_len <= 0) return TQ_ERR_INVALID_ARG;
    if (num_q_heads % c->num_kv_heads) return TQ_ERR_INVALID_ARG;
    if (max_seq_len < q_len) return TQ_ERR_INVALID_ARG;
    const int64_t need_pages = ((int64_t)max_seq_len + c->page_size - 1) / c->page_size;
    if (max_pages_per_seq < need_pages) return TQ_ERR_INVALID_ARG;
    const int64_t G = (int64_t)q_len * (num_q_heads / c->num_kv_heads);
    if (G > kMaxRows) return TQ_ERR_UNSUPPORTED;
    if (batch > 65535) return TQ_ERR_UNSUPPORTED;
    if ((int64_t)c->num_kv_heads * tq::decode_row_groups(c->format, (int)G) > 65535)
        return TQ_ERR_UNSUPPORTED;
    if (batch == 0) return TQ_OK;
    if (!q || !page_table || !seq_lens || !out) return TQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(page_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return TQ_ERR_INVALID_ARG;
    return TQ_OK;
}

// Bytes of one K (or V) block; 0 for an unsupported combination.
int64_t cache_block_bytes(int32_t format, int32_t head_dim, int32_t page_size)
{
    return block_bytes(format, head_dim, page_size);
}

}  // namespace tq

namespace {

tq_status check_decode(const void* q, const tq_cache* c, const int32_t* page_table,
                       int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                       int32_t q_len, int32_t num_q_heads, int32_t max_seq_len, const float* out,
                       const void* workspace, size_t workspace_bytes, bool turbo)
{
    tq_status s = tq::check_decode_call(q, c, page_table, max_pages_per_seq, seq_lens, batch,
                                        q_len, num_q_heads, max_seq_len, out, turbo);
    if (s != TQ_OK || batch == 0) return s;
    const int64_t G = (int64_t)q_len * (num_q_heads / c->num_kv_heads);
    const size_t need = tq::decode_workspace_bytes(batch, c->num_kv_heads, (int)G, max_seq_len,
                                                   c->page_size, c->format);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return TQ_ERR_WORKSPACE;
        if (!aligned16(workspace)) return TQ_ERR_INVALID_ARG;
    }
    return TQ_OK;
}

tq_status decode_common(const void* q, const tq_cache* cache, const int32_t* page_table,
                        int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                        int32_t q_len, int32_t num_q_heads, int32_t max_seq_len, float* out,
                        void* workspace, size_t workspace_bytes, void* stream, bool turbo)
{
    tq_status s = check_decode(q, cache, page_table, max_pages_per_seq, seq_lens, batch, q_len,
                               num_q_heads, max_seq_len, out, workspace, workspace_bytes, turbo);
    if (s != TQ_OK || batch == 0) return s;
    return from_cuda(tq::launch_decode(q, *cache, block_bytes(cache->format, 128, cache->page_size),
                                       page_table, max_pages_per_seq, seq_lens, batch, q_len,
                                       num_q_heads, max_seq_len, out, workspace,
                                       static_cast<cudaStream_t>(stream)));
}

}  // namespace

TQ_API int32_t tq_abi_version(void) { return TQ_ABI_VERSION; }

TQ_API const char* tq_status_string(tq_status status)
{
    switch (status) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT";
    case TQ_ERR_DEVICE_CHECK: return "TQ_ERR_DEVICE_CHECK";
    case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE";
    case TQ_ERR_NO_PAGES: return "TQ_ERR_NO_PAGES";
    default: return "TQ_ERR_UNKNOWN";
    }
}

TQ_API size_t tq_page_block_bytes(int32_t format, int32_t head_dim, int32_t page_size)
{
    return (size_t)block_bytes(format, head_dim, page_size);
}

TQ_API tq_status tq_quantize_append(const void* k, const void* v, const int64_t* slot_mapping,
                                    int32_t num_tokens, int32_t bits, const tq_cache* cache,
                                    void* stream)
{
    tq_status s = check_append(k, v, slot_mapping, num_tokens, cache, true);
    if (s != TQ_OK) return s;
    if (bits != cache->format) return TQ_ERR_INVALID_ARG;
    if (num_tokens == 0) return TQ_OK;
    return from_cuda(tq::launch_quantize_append(
        k, v, slot_mapping, num_tokens, bits, *cache,
        block_bytes(cache->format, 128, cache->page_size), static_cast<cudaStream_t>(stream)));
}

TQ_API tq_status tq_append_bf16(const void* k, const void* v, const int64_t* slot_mapping,
                                int32_t num_tokens, const tq_cache* cache, void* stream)
{
    tq_status s = check_append(k, v, slot_mapping, num_tokens, cache, false);
    if (s != TQ_OK || num_tokens == 0) return s;
    return from_cuda(tq::launch_append_bf16(k, v, slot_mapping, num_tokens, *cache,
                                            static_cast<cudaStream_t>(stream)));
}

TQ_API size_t tq_decode_workspace_size(int32_t batch, int32_t q_len, int32_t num_q_heads,
                                       int32_t max_seq_len, const tq_cache* cache)
{
    if (!cache || batch <= 0 || q_len <= 0 || num_q_heads <= 0 || max_seq_len <= 0) return 0;
    if (cache->num_kv_heads <= 0 || num_q_heads % cache->num_kv_heads) return 0;
    if (block_bytes(cache->format, cache->head_dim, cache->page_size) == 0) return 0;
    const int64_t G = (int64_t)q_len * (num_q_heads / cache->num_kv_heads);
    if (G > kMaxRows) return 0;
    return tq::decode_workspace_bytes(batch, cache->num_kv_heads, (int)G, max_seq_len,
                                      cache->page_size, cache->format);
}

TQ_API tq_status tq_decode_workspace_init(void* workspace, size_t workspace_bytes, void* stream)
{
    if (workspace_bytes == 0) return TQ_OK;
    if (!workspace) return TQ_ERR_INVALID_ARG;
    return from_cuda(cudaMemsetAsync(workspace, 0, workspace_bytes,
                                     static_cast<cudaStream_t>(stream)));
}

TQ_API tq_status tq_paged_decode(const void* q, const tq_cache* cache, const int32_t* page_table,
                                 int32_t max_pages_per_seq, const int32_t* seq_lens,
                                 int32_t batch, int32_t q_len, int32_t num_q_heads,
                                 int32_t max_seq_len, float* out, void* workspace,
                                 size_t workspace_bytes, void* stream)
{
    return decode_common(q, cache, page_table, max_pages_per_seq, seq_lens, batch, q_len,
                         num_q_heads, max_seq_len, out, workspace, workspace_bytes, stream, true);
}

TQ_API tq_status tq_paged_decode_bf16(const void* q, const tq_cache* cache,
                                      const int32_t* page_table, int32_t max_pages_per_seq,
                                      const int32_t* seq_lens, int32_t batch, int32_t q_len,
                                      int32_t num_q_heads, int32_t max_seq_len, float* out,
                                      void* workspace, size_t workspace_bytes, void* stream)
{
    return decode_common(q, cache, page_table, max_pages_per_seq, seq_lens, batch, q_len,
                         num_q_heads, max_seq_len, out, workspace, workspace_bytes, stream, false);
}

TQ_API tq_status tq_read_device_error(const tq_cache* cache, uint32_t* code, int32_t clear,
                                      void* stream)
{
    if (!cache || !code) return TQ_ERR_INVALID_ARG;
    *code = 0;
    if (!cache->dev_error) return TQ_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto deadline = std::chrono::steady_clock::now() + std::chrono::seconds(10);
    for (;;) {
        const cudaError_t q = cudaStreamQuery(s);
        if (q == cudaSuccess) break;
        if (q != cudaErrorNotReady) return TQ_ERR_CUDA;
        if (std::chrono::steady_clock::now() > deadline) return TQ_ERR_TIMEOUT;
        std::this_thread::sleep_for(std::chrono::microseconds(100));
    }
    uint32_t host = 0;
    cudaError_t e = cudaMemcpy(&host, cache->dev_error, sizeof host, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return TQ_ERR_CUDA;
    *code = host;
    if (clear) {
        e = cudaMemset(cache->dev_error, 0, sizeof(uint32_t));
        if (e != cudaSuccess) return TQ_ERR_CUDA;
    }
    return TQ_OK;
}

TQ_API tq_status tq_hbm_copy(const void* src, void* dst, size_t bytes, void* stream)
{
    if (bytes == 0) return TQ_OK;
    if (!src || !dst || !aligned16(src) || !aligned16(dst) || (bytes & 15u)) return TQ_ERR_INVALID_ARG;
    return from_cuda(tq::launch_hbm_copy(src, dst, bytes, static_cast<cudaStream_t>(stream)));
}

TQ_API tq_status tq_hbm_read(const void* src, size_t bytes, uint32_t* sink, void* stream)
{
    if (bytes == 0) return TQ_OK;
    if (!src || !sink || !aligned16(src) || (bytes & 15u)) return TQ_ERR_INVALID_ARG;
    return from_cuda(tq::launch_hbm_read(src, bytes, sink, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- graphs
struct tq_step_graph {
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
};

TQ_API tq_status tq_step_graph_create(const tq_cache* cache, const tq_step* step, void* stream,
                                      tq_step_graph** graph)
{
    if (!graph || !step || !stream) return TQ_ERR_INVALID_ARG;    // not the legacy stream
    *graph = nullptr;
    const tq_status sc = check_cache(cache, cache ? cache->format != TQ_BF16 : true);
    if (sc != TQ_OK) return sc;
    const bool turbo = cache->format != TQ_BF16;
    tq_status s = check_append(step->k, step->v, step->slot_mapping, step->num_tokens, cache, turbo);
    if (s != TQ_OK) return s;
    s = check_decode(step->q, cache, step->page_table, step->max_pages_per_seq, step->seq_lens,
                     step->batch, step->q_len, step->num_q_heads, step->max_seq_len, step->out,
                     step->workspace, step->workspace_bytes, turbo);
    if (s != TQ_OK) return s;
    tq_step_graph* g = new (std::nothrow) tq_step_graph();
    if (!g) return TQ_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // relaxed capture: a kernel's first launch on a device also sets its
    // shared-memory attribute, which this mode permits during capture
    cudaError_t e = cudaStreamBeginCapture(st, cudaStreamCaptureModeRelaxed);
    cudaError_t le = cudaSuccess;
    if (e == cudaSuccess) {
        const int64_t bb = block_bytes(cache->format, 128, cache->page_size);
        if (step->num_tokens > 0)
            le = turbo ? tq::launch_quantize_append(step->k, step->v, step->slot_mapping,
                                                    step->num_tokens, cache->format, *cache, bb, st)
                       : tq::launch_append_bf16(step->k, step->v, step->slot_mapping,
                                                step->num_tokens, *cache, st);
        if (le == cudaSuccess && step->batch > 0)
            le = tq::launch_decode(step->q, *cache, bb, step->page_table, step->max_pages_per_seq,
                                   step->seq_lens, step->batch, step->q_len, step->num_q_heads,
                                   step->max_seq_len, step->out, step->workspace, st);
        e = cudaStreamEndCapture(st, &g->graph);
    }
    if (e == cudaSuccess && le == cudaSuccess)
        e = cudaGraphInstantiate(&g->exec, g->graph, 0);
    if (e != cudaSuccess || le != cudaSuccess) {
        if (g->exec) cudaGraphExecDestroy(g->exec);
        if (g->graph) cudaGraphDestroy(g->graph);
        delete g;
        cudaGetLastError();                           // clear a launch error recorded in capture
        return TQ_ERR_CUDA;
    }
    *graph = g;
    return TQ_OK;
}

TQ_API tq_status tq_step_graph_launch(tq_step_graph* graph, void* stream)
{
    if (!graph || !graph->exec) return TQ_ERR_INVALID_ARG;
    return from_cuda(cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)));
}

TQ_API void tq_step_graph_destroy(tq_step_graph* graph)
{
    if (!graph) return;
    if (graph->exec) cudaGraphExecDestroy(graph->exec);
    if (graph->graph) cudaGraphDestroy(graph->graph);
    delete graph;
}
