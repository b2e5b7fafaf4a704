// Cache write (reshape_and_cache) and copy-on-write block copy kernels, plus
// the library's device-side error word.
//
// reshape_and_cache: a generated token's key and value rows go into the row
// its slot names ("vLLM内存管理与PagedAttention精讲" ch.2 §2.4.2, a new block
// only when the current one is full; "VLLM中PagedAttention如何降低显存碎片？"
// §四 flow: allocate a free page, update the mapping).  With the cache laid
// out [num_blocks][block_size][kv_heads][head_dim], slot s is one contiguous
// row of kv_heads * head_dim elements, so the write is a 16-byte-vector row
// copy.
//
// copy_blocks: copy-on-write of a shared block ("vLLM内存管理与PagedAttention
// 精讲" §2.4.3): block dst <- block src for keys and values; a block is one
// contiguous run of block_size * kv_heads * head_dim elements.
#include "common.cuh"
#include "internal.h"

namespace pa {

__device__ unsigned g_device_error_word;

namespace {

__global__ void __launch_bounds__(128)
    reshape_and_cache_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                             uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                             const int64_t* __restrict__ slots, int num_tokens, int row_vecs,
                             int64_t num_slots, unsigned* err) {
    pdl_wait();
    pdl_launch_dependents();
    for (int t = blockIdx.x; t < num_tokens; t += gridDim.x) {
        const int64_t s = slots[t];
        if (s < 0) continue;
        if (s >= num_slots) {
            if (threadIdx.x == 0) raise_error(err, PA_DEVERR_SLOT);
            continue;
        }
        const uint4* ks = key + (size_t)t * row_vecs;
        const uint4* vs = value + (size_t)t * row_vecs;
        uint4* kd = k_cache + (size_t)s * row_vecs;
        uint4* vd = v_cache + (size_t)s * row_vecs;
        for (int i = threadIdx.x; i < row_vecs; i += blockDim.x) {
            kd[i] = ks[i];
            vd[i] = vs[i];
        }
    }
}

// Block dst of the destination pool <- block src of the source pool, keys and
// values; the pools are the same cache (copy-on-write) or a device cache and
// a pinned host cache reached through its device-mapped address (swapping).
__global__ void __launch_bounds__(256)
    move_blocks_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                       const uint4* __restrict__ src_k, const uint4* __restrict__ src_v,
                       const int64_t* __restrict__ mapping, int64_t block_vecs, int src_blocks,
                       int dst_blocks, unsigned err_bits, unsigned* err) {
    pdl_wait();
    pdl_launch_dependents();
    const int pair = blockIdx.x;
    const int64_t src = mapping[2 * pair], dst = mapping[2 * pair + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0) raise_error(err, err_bits);
        return;
    }
    const uint4* ks = src_k + src * block_vecs;
    const uint4* vs = src_v + src * block_vecs;
    uint4* kd = dst_k + dst * block_vecs;
    uint4* vd = dst_v + dst * block_vecs;
    for (int64_t i = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; i < block_vecs;
         i += (int64_t)gridDim.y * blockDim.x) {
        kd[i] = ks[i];
        vd[i] = vs[i];
    }
}

// The mapping update of one decode step: sequence s's newest token (position
// context_lens[s] - 1) sits in slot slot_mapping[s], so table entry
// (context_lens[s] - 1) / block_size becomes slot / block_size -- a new
// block, a copy-on-write replacement, or the entry it already holds.
__global__ void __launch_bounds__(256)
    update_tables_kernel(int32_t* __restrict__ tables, int stride,
                         const int32_t* __restrict__ lens, const int64_t* __restrict__ slots,
                         int num_seqs, int block_size, int num_blocks, unsigned* err) {
    pdl_wait();
    pdl_launch_dependents();
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= num_seqs) return;
    const int64_t slot = slots[s];
    if (slot < 0) return;
    const int pos = lens[s] - 1;
    const int64_t blk = slot / block_size;
    if (pos < 0 || pos / block_size >= stride || blk >= num_blocks) {
        raise_error(err, PA_DEVERR_SLOT);
        return;
    }
    tables[(size_t)s * stride + pos / block_size] = (int32_t)blk;
}

}  // namespace

pa_status launch_update_tables(int32_t* tables, int stride, const int32_t* lens,
                               const int64_t* slots, int num_seqs, int block_size,
                               int num_blocks, cudaStream_t stream) {
    if (num_seqs == 0) return PA_OK;
    unsigned* err = device_error_word();
    if (!err) return fail(PA_ERR_CUDA, "device error word unavailable");
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((num_seqs + 255) / 256);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    add_pdl_attr(attr, &cfg.numAttrs);
    cudaError_t e = cudaLaunchKernelEx(&cfg, update_tables_kernel, tables, stride, lens, slots,
                                       num_seqs, block_size, num_blocks, err);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "table update launch: %s", cudaGetErrorString(e));
    return PA_OK;
}

unsigned* device_error_word() {
    static unsigned* cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!cached[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
        cached[dev] = static_cast<unsigned*>(p);
    }
    return cached[dev];
}

int num_sms() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

pa_status launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                   void* v_cache, const int64_t* slots, int num_tokens,
                                   int64_t row_bytes, int64_t num_slots, cudaStream_t stream) {
    if (num_tokens == 0) return PA_OK;
    unsigned* err = device_error_word();
    if (!err) return fail(PA_ERR_CUDA, "device error word unavailable");
    const int grid = num_tokens < 8 * num_sms() ? num_tokens : 8 * num_sms();
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(128);
    cfg.stream = stream;
    cfg.attrs = attr;
    add_pdl_attr(attr, &cfg.numAttrs);
    cudaError_t e = cudaLaunchKernelEx(
        &cfg, reshape_and_cache_kernel, static_cast<const uint4*>(key),
        static_cast<const uint4*>(value), static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache), slots, num_tokens, (int)(row_bytes / 16), num_slots, err);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "reshape_and_cache launch: %s", cudaGetErrorString(e));
    return PA_OK;
}

pa_status launch_move_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                             const int64_t* mapping, int num_pairs, int64_t block_bytes,
                             int src_blocks, int dst_blocks, unsigned err_bits,
                             cudaStream_t stream) {
    if (num_pairs == 0) return PA_OK;
    unsigned* err = device_error_word();
    if (!err) return fail(PA_ERR_CUDA, "device error word unavailable");
    const int64_t vecs = block_bytes / 16;
    int chunks = (int)(vecs / 1024);
    chunks = chunks < 1 ? 1 : (chunks > 32 ? 32 : chunks);
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_pairs, chunks);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    add_pdl_attr(attr, &cfg.numAttrs);
    cudaError_t e = cudaLaunchKernelEx(
        &cfg, move_blocks_kernel, static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v),
        static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v), mapping, vecs,
        src_blocks, dst_blocks, err_bits, err);
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "block move launch: %s", cudaGetErrorString(e));
    return PA_OK;
}

pa_status launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* mapping, int num_pairs,
                             int64_t block_bytes, int num_blocks, cudaStream_t stream) {
    return launch_move_blocks(k_cache, v_cache, k_cache, v_cache, mapping, num_pairs, block_bytes,
                              num_blocks, num_blocks, PA_DEVERR_COPY_ID, stream);
}

}  // namespace pa
