// pa_decode_split_noalloc: split-K decode for callers that cannot allocate
// device memory.
//
// pa_decode_split needs a workspace for the per-partition maxima, sums and
// partial outputs, and expects the caller to allocate it.  Some callers
// cannot: a plugin running inside a host framework that owns all device
// memory and hands plugins none, or a serving process with a fixed memory
// budget that forbids any device allocation after start-up.  This entry
// point takes the same arguments minus the workspace and uses a fixed-size
// scratch array that lives in the library itself instead.
//
// The scratch is a file-scope __device__ array of PA_NOALLOC_SCRATCH_BYTES;
// every GPU that loads this library's module holds it until the process
// exits.  Host code cannot use the array's name as a device address (in host
// code it names a host-side stand-in), so the first call on each device, with
// that device current, looks up the real address with cudaGetSymbolAddress
// and caches it.  That first call should come before any stream capture.
// All calls share the one array and it keeps whatever the last call left in
// it; nothing in it needs to start at zero, because the partition kernel
// writes every slot the merge kernel reads within the same call.  Calls that
// overlap on the GPU (on different streams, or from different host threads)
// race on the array and corrupt each other's results.
#include <mutex>

#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device (set up once
// per device).  Returns PA_OK and the address, or an error status.
pa_status scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return pa::fail(PA_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kMaxDevices - 1);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return pa::fail(PA_ERR_CUDA, "cudaGetSymbolAddress of the decode scratch: %s",
                            cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_split_noalloc(
    void* out_d, const void* q_d, const void* k_cache_d, const void* v_cache_d,
    const int32_t* block_tables_d, int max_blocks_per_seq, const int32_t* context_lens_d,
    int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
    float scale, pa_dtype dtype, int max_context_len, int partition_size, pa_stream_t stream) {
    const size_t need = pa_decode_split_workspace_bytes(num_seqs, num_heads, head_dim,
                                                        max_context_len, partition_size);
    if (need > (size_t)PA_NOALLOC_SCRATCH_BYTES)
        return pa::fail(PA_ERR_UNSUPPORTED,
                        "this batch needs %zu bytes of decode scratch; the built-in scratch "
                        "holds %d bytes (use pa_decode_split with a caller workspace)",
                        need, PA_NOALLOC_SCRATCH_BYTES);
    if (num_seqs == 0)
        return pa_decode_split(out_d, q_d, k_cache_d, v_cache_d, block_tables_d,
                               max_blocks_per_seq, context_lens_d, num_seqs, num_heads,
                               num_kv_heads, head_dim, block_size, num_blocks, scale, dtype,
                               max_context_len, partition_size, nullptr, 0, stream);
    void* scratch = nullptr;
    if (pa_status s = scratch_address(&scratch)) return s;
    return pa_decode_split(out_d, q_d, k_cache_d, v_cache_d, block_tables_d, max_blocks_per_seq,
                           context_lens_d, num_seqs, num_heads, num_kv_heads, head_dim,
                           block_size, num_blocks, scale, dtype, max_context_len, partition_size,
                           scratch, (size_t)PA_NOALLOC_SCRATCH_BYTES, stream);
}
