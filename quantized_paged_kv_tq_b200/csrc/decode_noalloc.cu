// tq_paged_decode_noalloc: the turbo decode with its scratch in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// Who needs it: code that is not allowed to allocate device memory once it
// is running -- for example a plugin whose enqueue hook an inference runtime
// calls with a fixed memory plan, or a service that reserves all device
// memory at start-up and treats any later cudaMalloc as an error.  Such
// callers still own q, the cache, the page table and the output; this entry
// point only removes the split-KV workspace from what they must provide.
//
// Cost and limits: the array below is kStaticScratchBytes (64 MiB) on every
// GPU that loads libtq.so, held until the process exits.  Shapes whose
// workspace would exceed it are rejected with TQ_ERR_WORKSPACE before any
// launch.  All calls share the one array, so calls that overlap in time on
// the GPU (different streams, or different host threads, on one device)
// race on it; callers must serialise them.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/tq.h"

#define TQ_API extern "C" __attribute__((visibility("default")))

namespace tq {
tq_status check_decode_call(const void* q, const tq_cache* c, const int32_t* page_table,
                            int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                            int32_t q_len, int32_t num_q_heads, int32_t max_seq_len,
                            const float* out, bool turbo);
int64_t cache_block_bytes(int32_t format, int32_t head_dim, int32_t page_size);
size_t decode_workspace_bytes(int batch, int num_kv_heads, int G, int max_seq_len,
                              int page_size, int format);
int decode_row_groups(int format, int G);
cudaError_t launch_decode(const void* q, const tq_cache& c, int64_t block_bytes,
                          const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                          int batch, int q_len, int num_q_heads, int max_seq_len, float* out,
                          void* workspace, cudaStream_t stream);
}  // namespace tq

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

// The scratch itself.  Host code must never pass this symbol to a kernel: on
// the host it only names the variable; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (the first call on a device does this; it should therefore happen
// before any stream capture that includes this entry point).
cudaError_t scratch_on_current_device(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

TQ_API tq_status tq_paged_decode_noalloc(const void* q, const tq_cache* cache,
                                         const int32_t* page_table, int32_t max_pages_per_seq,
                                         const int32_t* seq_lens, int32_t batch, int32_t q_len,
                                         int32_t num_q_heads, int32_t max_seq_len, float* out,
                                         void* stream)
{
    // the same host checks as tq_paged_decode (one shared function), then
    // the scratch-size limit in place of the workspace checks
    const tq_status st = tq::check_decode_call(q, cache, page_table, max_pages_per_seq, seq_lens,
                                               batch, q_len, num_q_heads, max_seq_len, out, true);
    if (st != TQ_OK || batch == 0) return st;
    const int f = cache->format;
    const int64_t G = (int64_t)q_len * (num_q_heads / cache->num_kv_heads);

    const size_t need = tq::decode_workspace_bytes(batch, cache->num_kv_heads, (int)G,
                                                   max_seq_len, cache->page_size, f);
    if (need > kStaticScratchBytes) return TQ_ERR_WORKSPACE;   // beyond the fixed maximum

    void* scratch = nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (need > 0) {
        if (scratch_on_current_device(&scratch) != cudaSuccess) return TQ_ERR_CUDA;
        // The array keeps whatever the previous call left.  Only the merge
        // counters at its start must begin at zero; the partials are always
        // written before they are read.
        const size_t units =
            (size_t)batch * cache->num_kv_heads * tq::decode_row_groups(f, (int)G);
        if (cudaMemsetAsync(scratch, 0, units * sizeof(uint32_t), s) != cudaSuccess)
            return TQ_ERR_CUDA;
    }
    const int64_t block = tq::cache_block_bytes(f, cache->head_dim, cache->page_size);
    const cudaError_t e = tq::launch_decode(q, *cache, block, page_table, max_pages_per_seq,
                                            seq_lens, batch, q_len, num_q_heads, max_seq_len,
                                            out, scratch, s);
    return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
