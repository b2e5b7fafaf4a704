// C ABI of libpagedattn.so: argument checks, optional host-side index
// validation, tensor-map encoding and dispatch to the kernel instances.
// The public contract of every call is documented in include/pagedattn.h.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_set>
#include <vector>

#include <cudaTypedefs.h>

#include "launch.cuh"

namespace pa {

namespace {

thread_local std::string g_last_error;
// process-wide options, read and set from any host thread
std::atomic<int> g_validate{-1};     // -1: read PA_VALIDATE on first use
std::atomic<int> g_decode_ctas{0};   // 0: automatic
std::atomic<int> g_pdl{-1};          // -1: read PA_PDL on first use (default on)
std::atomic<int> g_wait_us{(int)(WAIT_LIMIT_NS / 1000)};   // limit of every pipeline wait
std::atomic<int> g_underfed{0};      // test only: stage barriers armed above their loads

bool validate_enabled() {
    int v = g_validate.load(std::memory_order_relaxed);
    if (v < 0) {
        const char* e = std::getenv("PA_VALIDATE");
        int want = (e && e[0] && e[0] != '0') ? 1 : 0;
        // an explicit pa_set_option set since then wins
        g_validate.compare_exchange_strong(v, want);
        v = g_validate.load(std::memory_order_relaxed);
    }
    return v == 1;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Encoded tensor maps, keyed by everything the encoding depends on (base
// address, data type, sizes, box, swizzle): a hit returns the same 128 bytes
// a fresh cuTensorMapEncodeTiled would, and saves the encode on every launch
// over the same cache or query buffer.  A small round-robin cache, shared by
// all host threads under a mutex.
struct MapKey {
    const void* base;
    int kind;                      // 0: cache tensor, 1: query tensor
    int v[7];
    bool operator==(const MapKey& o) const {
        if (base != o.base || kind != o.kind) return false;
        for (int i = 0; i < 7; ++i)
            if (v[i] != o.v[i]) return false;
        return true;
    }
};
constexpr int MAP_CACHE = 32;
std::mutex g_map_mutex;
MapKey g_map_keys[MAP_CACHE];
CUtensorMap g_maps[MAP_CACHE];
int g_map_count = 0, g_map_next = 0;

bool map_lookup(const MapKey& k, CUtensorMap* out) {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    for (int i = 0; i < g_map_count; ++i)
        if (g_map_keys[i] == k) {
            *out = g_maps[i];
            return true;
        }
    return false;
}

void map_store(const MapKey& k, const CUtensorMap& m) {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    for (int i = 0; i < g_map_count; ++i)
        if (g_map_keys[i] == k) return;
    const int i = g_map_count < MAP_CACHE ? g_map_count++ : g_map_next;
    g_map_next = (i + 1) % MAP_CACHE;
    g_map_keys[i] = k;
    g_maps[i] = m;
}

int elem_size(pa_dtype dt) { return dt == PA_DTYPE_F32 ? 4 : 2; }

pa_status check_geometry(pa_dtype dt, int head_dim, int block_size) {
    if (dt != PA_DTYPE_F32 && dt != PA_DTYPE_BF16)
        return fail(PA_ERR_UNSUPPORTED, "dtype %d not supported", (int)dt);
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return fail(PA_ERR_UNSUPPORTED, "head_dim %d not built (64, 128, 256)", head_dim);
    if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64 &&
        block_size != 128)
        return fail(PA_ERR_UNSUPPORTED, "block_size %d not built (8, 16, 32, 64, 128)", block_size);
    return PA_OK;
}

template <typename T>
bool copy_to_host(std::vector<T>& dst, const T* src, size_t n, cudaStream_t stream) {
    dst.resize(n);
    if (n == 0) return true;
    if (cudaMemcpyAsync(dst.data(), src, n * sizeof(T), cudaMemcpyDeviceToHost, stream) !=
        cudaSuccess)
        return false;
    return cudaStreamSynchronize(stream) == cudaSuccess;
}

// Every sequence's length fits its table row and the entries it reads are
// blocks of the pool (host copies of the tables and lengths).
pa_status check_tables(const std::vector<int32_t>& t, const std::vector<int32_t>& l,
                       int max_blocks, int num_seqs, int block_size, int num_blocks) {
    for (int s = 0; s < num_seqs; ++s) {
        if (l[s] < 0 || (int64_t)l[s] > (int64_t)max_blocks * block_size)
            return fail(PA_ERR_BAD_BLOCK_ID, "context_lens[%d] = %d outside [0, %lld]", s, l[s],
                        (long long)max_blocks * block_size);
        const int n = (l[s] + block_size - 1) / block_size;
        for (int j = 0; j < n; ++j) {
            const int32_t b = t[(size_t)s * max_blocks + j];
            if (b < 0 || b >= num_blocks)
                return fail(PA_ERR_BAD_BLOCK_ID, "block_tables[%d, %d] = %d outside [0, %d)", s, j,
                            b, num_blocks);
        }
    }
    return PA_OK;
}

pa_status validate_decode(const int32_t* tables, int max_blocks, const int32_t* lens, int num_seqs,
                          int block_size, int num_blocks, cudaStream_t stream) {
    std::vector<int32_t> t, l;
    if (!copy_to_host(l, lens, (size_t)num_seqs, stream) ||
        !copy_to_host(t, tables, (size_t)num_seqs * max_blocks, stream))
        return fail(PA_ERR_CUDA, "validation copy failed");
    return check_tables(t, l, max_blocks, num_seqs, block_size, num_blocks);
}

pa_status check_decode_args(void* out, const void* q, const void* kc, const void* vc,
                            const int32_t* tables, int max_blocks, const int32_t* lens,
                            int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                            int block_size, int num_blocks, pa_dtype dt, float scale) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks <= 0)
        return fail(PA_ERR_INVALID_ARG, "sizes must be positive (num_seqs >= 0)");
    if (num_seqs > 65535) return fail(PA_ERR_UNSUPPORTED, "num_seqs above 65535");
    if (num_heads % num_kv_heads != 0)
        return fail(PA_ERR_INVALID_ARG, "num_heads %d is not a multiple of num_kv_heads %d",
                    num_heads, num_kv_heads);
    if (num_kv_heads > 65535) return fail(PA_ERR_UNSUPPORTED, "num_kv_heads above 65535");
    if ((int64_t)max_blocks * block_size > 0x7fffffff)
        return fail(PA_ERR_UNSUPPORTED, "max_blocks_per_seq * block_size overflows int32");
    if (pa_status s = check_geometry(dt, head_dim, block_size)) return s;
    const int g = num_heads / num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8)
        return fail(PA_ERR_UNSUPPORTED, "group size %d not built (1, 2, 4, 8)", g);
    if (!(scale == scale)) return fail(PA_ERR_INVALID_ARG, "scale is NaN");
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !kc || !vc || !tables || !lens)
        return fail(PA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(out) || !aligned16(q) || !aligned16(kc) || !aligned16(vc))
        return fail(PA_ERR_INVALID_ARG, "q, out and caches must be 16-byte aligned");
    return PA_OK;
}

// CTAs per (sequence, kv head) for pa_decode.  Splitting costs a cluster
// merge and shortens every CTA's stream, so it only pays when the grid
// would otherwise leave SMs idle: grow the cluster while there are fewer
// (sequence, kv head) pairs than two per SM and each CTA keeps at least
// 1024 tokens of its sequence's capacity.
int auto_decode_ctas(int num_seqs, int num_kv_heads, int max_blocks, int block_size) {
    const int64_t max_tokens = (int64_t)max_blocks * block_size;
    const int64_t work = (int64_t)num_seqs * num_kv_heads;
    const int64_t target = 2LL * num_sms();
    int c = 1;
    while (c < 8 && work * c < target && max_tokens / (2 * c) >= 1024) c *= 2;
    return c;
}

pa_status dispatch_decode(const DecodeLaunch& l, pa_dtype dt, int head_dim) {
    if (dt == PA_DTYPE_F32) {
        if (head_dim == 64) return launch_decode_f32_d64(l);
        if (head_dim == 128) return launch_decode_f32_d128(l);
        return launch_decode_f32_d256(l);
    }
    if (head_dim == 64) return launch_decode_bf16_d64(l);
    if (head_dim == 128) return launch_decode_bf16_d128(l);
    return launch_decode_bf16_d256(l);
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// The device error word and the pipeline-wait settings every decode launch carries.
pa_status set_error_and_waits(DecodeArgs& args) {
    args.err = device_error_word();
    if (!args.err) return fail(PA_ERR_CUDA, "device error word unavailable");
    args.wait_ns = 1000ull * (unsigned long long)g_wait_us.load(std::memory_order_relaxed);
    args.tx_extra = g_underfed.load(std::memory_order_relaxed) ? 16u : 0u;
    return PA_OK;
}

// Chunks of partitions per (sequence, head) in the log-sum-exp reduce: enough
// CTAs to fill the GPU a few times over (a fixed target, so the workspace
// size does not depend on the device), at least 16 partitions per chunk.
int reduce_chunks(size_t heads, size_t parts) {
    constexpr size_t TARGET_CTAS = 600;
    size_t c = (TARGET_CTAS + heads - 1) / heads;
    const size_t most = (parts + 15) / 16;
    if (c > most) c = most;
    return c < 1 ? 1 : (int)c;
}

}  // namespace

bool pdl_enabled() {
    int v = g_pdl.load(std::memory_order_relaxed);
    if (v < 0) {
        const char* e = std::getenv("PA_PDL");
        int want = (e && e[0] == '0') ? 0 : 1;
        g_pdl.compare_exchange_strong(v, want);
        v = g_pdl.load(std::memory_order_relaxed);
    }
    return v == 1;
}

void add_pdl_attr(cudaLaunchAttribute* attrs, unsigned* n) {
    if (!pdl_enabled()) return;
    attrs[*n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[*n].val.programmaticStreamSerializationAllowed = 1;
    ++*n;
}

pa_status fail(pa_status status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

pa_status encode_cache_map(CUtensorMap* map, const void* base, pa_dtype dtype, int head_dim,
                           int num_kv_heads, int block_size, int num_blocks, int box_inner,
                           int rows, bool swizzle128) {
    const MapKey key{base, 0, {(int)dtype, head_dim, num_kv_heads, block_size, num_blocks,
                               box_inner * 1024 + rows, swizzle128 ? 1 : 0}};
    if (map_lookup(key, map)) return PA_OK;
    auto enc = tensor_map_encoder();
    if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t es = (cuuint64_t)elem_size(dtype);
    cuuint64_t dims[4] = {(cuuint64_t)head_dim, (cuuint64_t)num_kv_heads, (cuuint64_t)block_size,
                          (cuuint64_t)num_blocks};
    cuuint64_t strides[3] = {head_dim * es, (cuuint64_t)num_kv_heads * head_dim * es,
                             (cuuint64_t)block_size * num_kv_heads * head_dim * es};
    cuuint32_t box[4] = {(cuuint32_t)box_inner, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map,
                     dtype == PA_DTYPE_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                           : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    map_store(key, *map);
    return PA_OK;
}

pa_status encode_query_map(CUtensorMap* map, const void* q, int head_dim, int num_heads,
                           int num_seqs, int heads, int seqs) {
    const MapKey key{q, 1, {head_dim, num_heads, num_seqs, heads, seqs, 0, 0}};
    if (map_lookup(key, map)) return PA_OK;
    auto enc = tensor_map_encoder();
    if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_heads, (cuuint64_t)num_seqs};
    cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)num_heads * head_dim * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)heads, (cuuint32_t)seqs};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled (queries) failed (%d)", (int)r);
    map_store(key, *map);
    return PA_OK;
}

}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_last_error(void) { return g_last_error.c_str(); }

const char* pa_status_string(pa_status s) {
    switch (s) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARG: return "invalid argument";
        case PA_ERR_UNSUPPORTED: return "unsupported configuration";
        case PA_ERR_OUT_OF_BLOCKS: return "out of blocks";
        case PA_ERR_BAD_BLOCK_ID: return "bad block id";
        case PA_ERR_CUDA: return "cuda error";
        case PA_ERR_DEVICE_CHECK: return "device check failed";
    }
    return "unknown status";
}

int pa_version(void) { return 1; }

pa_status pa_set_option(pa_option option, int value) {
    switch (option) {
        case PA_OPT_VALIDATE: g_validate = value ? 1 : 0; return PA_OK;
        case PA_OPT_PDL: g_pdl = value ? 1 : 0; return PA_OK;
        case PA_OPT_DECODE_SPLIT_CTAS:
            if (value != 0 && value != 1 && value != 2 && value != 4 && value != 8)
                return fail(PA_ERR_INVALID_ARG, "CTAs per (sequence, kv head) must be 0,1,2,4,8");
            g_decode_ctas = value;
            return PA_OK;
        case PA_OPT_WAIT_LIMIT_US:
            if (value < 100 || value > 10000000)
                return fail(PA_ERR_INVALID_ARG, "wait limit must be 100 .. 10000000 us");
            g_wait_us = value;
            return PA_OK;
        case PA_OPT_TEST_UNDERFED_STAGES: g_underfed = value ? 1 : 0; return PA_OK;
    }
    return fail(PA_ERR_INVALID_ARG, "unknown option %d", (int)option);
}

int pa_get_option(pa_option option) {
    switch (option) {
        case PA_OPT_VALIDATE: return validate_enabled() ? 1 : 0;
        case PA_OPT_DECODE_SPLIT_CTAS: return g_decode_ctas.load();
        case PA_OPT_PDL: return pdl_enabled() ? 1 : 0;
        case PA_OPT_WAIT_LIMIT_US: return g_wait_us.load();
        case PA_OPT_TEST_UNDERFED_STAGES: return g_underfed.load();
    }
    return -1;
}

pa_status pa_device_error(pa_stream_t stream, uint32_t* flags, int clear) {
    if (!flags) return fail(PA_ERR_INVALID_ARG, "null flags");
    unsigned* word = device_error_word();
    if (!word) return fail(PA_ERR_CUDA, "device error word unavailable");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    unsigned v = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
        return fail(PA_ERR_CUDA, "reading the device error word: %s",
                    cudaGetErrorString(cudaGetLastError()));
    *flags = v;
    if (clear && v && cudaMemset(word, 0, sizeof(unsigned)) != cudaSuccess)
        return fail(PA_ERR_CUDA, "clearing the device error word failed");
    if (v) return fail(PA_ERR_DEVICE_CHECK, "device error word 0x%x", v);
    return PA_OK;
}

pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                               pa_stream_t stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0)
        return fail(PA_ERR_INVALID_ARG, "sizes must be positive (num_tokens >= 0)");
    if (pa_status s = check_geometry(dtype, head_dim, block_size)) return s;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping)
        return fail(PA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_INVALID_ARG, "rows and caches must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t num_slots = (int64_t)num_blocks * block_size;
    if (validate_enabled()) {
        std::vector<int64_t> sl;
        if (!copy_to_host(sl, slot_mapping, (size_t)num_tokens, st))
            return fail(PA_ERR_CUDA, "validation copy failed");
        std::unordered_set<int64_t> seen;
        for (int t = 0; t < num_tokens; ++t) {
            if (sl[t] < -1 || sl[t] >= num_slots)
                return fail(PA_ERR_BAD_BLOCK_ID, "slot_mapping[%d] = %lld outside [-1, %lld)", t,
                            (long long)sl[t], (long long)num_slots);
            if (sl[t] >= 0 && !seen.insert(sl[t]).second)
                return fail(PA_ERR_BAD_BLOCK_ID, "slot %lld written twice", (long long)sl[t]);
        }
    }
    const int64_t row_bytes = (int64_t)num_kv_heads * head_dim * elem_size(dtype);
    return launch_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, num_tokens,
                                    row_bytes, num_slots, st);
}

}  // extern "C"

namespace {

// pa_decode, optionally with the fused append of one new token per sequence.
pa_status decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                      int head_dim, int block_size, int num_blocks, float scale, pa_dtype dtype,
                      const void* new_k, const void* new_v, const int64_t* new_slots,
                      int32_t* table_out, pa_stream_t stream) {
    if (pa_status s = check_decode_args(out, q, k_cache, v_cache, block_tables,
                                        max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                        num_kv_heads, head_dim, block_size, num_blocks, dtype,
                                        scale))
        return s;
    if (num_seqs == 0) return PA_OK;
    const bool append = new_slots != nullptr;
    if (append && (!new_k || !new_v || !aligned16(new_k) || !aligned16(new_v)))
        return fail(PA_ERR_INVALID_ARG, "key and value rows must be 16-byte aligned device pointers");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (validate_enabled() && table_out) {
        // the tables as the step leaves them: each new slot's block at its
        // sequence's last position, the slot on the new token's row
        std::vector<int32_t> t, l;
        std::vector<int64_t> sl;
        if (!copy_to_host(l, context_lens, (size_t)num_seqs, st) ||
            !copy_to_host(t, block_tables, (size_t)num_seqs * max_blocks_per_seq, st) ||
            !copy_to_host(sl, new_slots, (size_t)num_seqs, st))
            return fail(PA_ERR_CUDA, "validation copy failed");
        const int64_t num_slots = (int64_t)num_blocks * block_size;
        for (int s = 0; s < num_seqs; ++s) {
            if (sl[s] < 0) continue;
            const int pos = l[s] - 1;
            if (sl[s] >= num_slots || pos < 0 || (int64_t)pos >= (int64_t)max_blocks_per_seq * block_size ||
                sl[s] % block_size != pos % block_size)
                return fail(PA_ERR_BAD_BLOCK_ID,
                            "new slot of sequence %d is %lld, not row %d of a pool block", s,
                            (long long)sl[s], pos < 0 ? -1 : pos % block_size);
            t[(size_t)s * max_blocks_per_seq + pos / block_size] = (int32_t)(sl[s] / block_size);
        }
        if (pa_status s = check_tables(t, l, max_blocks_per_seq, num_seqs, block_size, num_blocks))
            return s;
    } else if (validate_enabled()) {
        if (pa_status s = validate_decode(block_tables, max_blocks_per_seq, context_lens,
                                          num_seqs, block_size, num_blocks, st))
            return s;
        if (append) {
            std::vector<int32_t> t, l;
            std::vector<int64_t> sl;
            if (!copy_to_host(l, context_lens, (size_t)num_seqs, st) ||
                !copy_to_host(t, block_tables, (size_t)num_seqs * max_blocks_per_seq, st) ||
                !copy_to_host(sl, new_slots, (size_t)num_seqs, st))
                return fail(PA_ERR_CUDA, "validation copy failed");
            for (int s = 0; s < num_seqs; ++s) {
                if (sl[s] < 0) continue;
                const int pos = l[s] - 1;
                const int64_t want =
                    pos < 0 ? -2
                            : (int64_t)t[(size_t)s * max_blocks_per_seq + pos / block_size] *
                                      block_size + pos % block_size;
                if (sl[s] != want)
                    return fail(PA_ERR_BAD_BLOCK_ID,
                                "new slot of sequence %d is %lld, its last position is slot %lld",
                                s, (long long)sl[s], (long long)want);
            }
        }
    }
    DecodeLaunch l = {};
    l.args.out = out;
    l.args.q = q;
    l.args.block_tables = block_tables;
    l.args.context_lens = context_lens;
    if (pa_status s = set_error_and_waits(l.args)) return s;
    l.args.scale_log2 = scale * 1.4426950408889634f;
    l.args.num_seqs = num_seqs;
    l.args.max_blocks = max_blocks_per_seq;
    l.args.max_tokens = max_blocks_per_seq * block_size;
    l.args.num_heads = num_heads;
    l.args.num_kv_heads = num_kv_heads;
    l.args.num_blocks = num_blocks;
    l.args.new_k = new_k;
    l.args.new_v = new_v;
    l.args.new_slots = new_slots;
    l.args.table_out = table_out;
    l.args.k_cache = const_cast<void*>(k_cache);
    l.args.v_cache = const_cast<void*>(v_cache);
    l.k_cache = k_cache;
    l.v_cache = v_cache;
    l.num_seqs = num_seqs;
    l.num_kv_heads = num_kv_heads;
    l.block_size = block_size;
    l.group = num_heads / num_kv_heads;
    const int ctas_opt = g_decode_ctas.load(std::memory_order_relaxed);
    l.ctas = ctas_opt ? ctas_opt
                           : auto_decode_ctas(num_seqs, num_kv_heads, max_blocks_per_seq,
                                              block_size);
    // one CTA per item: a longest-first grid; several CTAs per item: one
    // cluster per (sequence, kv head)
    l.args.sched = l.ctas > 1 ? SCHED_CLUSTER : SCHED_LPT;
    l.split = false;
    l.stream = st;
    return dispatch_decode(l, dtype, head_dim);
}

}  // namespace

extern "C" {

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int max_blocks_per_seq,
                    const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                    int head_dim, int block_size, int num_blocks, float scale, pa_dtype dtype,
                    pa_stream_t stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       scale, dtype, nullptr, nullptr, nullptr, nullptr, stream);
}

pa_status pa_decode_append(void* out, const void* q, const void* key, const void* value,
                           void* k_cache, void* v_cache, const int64_t* slot_mapping,
                           const int32_t* block_tables, int max_blocks_per_seq,
                           const int32_t* context_lens, int num_seqs, int num_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           float scale, pa_dtype dtype, pa_stream_t stream) {
    if (num_seqs > 0 && !slot_mapping) return fail(PA_ERR_INVALID_ARG, "null slot_mapping");
    return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       scale, dtype, key, value, slot_mapping, nullptr, stream);
}

pa_status pa_decode_step(void* out, const void* q, const void* key, const void* value,
                         void* k_cache, void* v_cache, const int64_t* slot_mapping,
                         int32_t* block_tables, int max_blocks_per_seq,
                         const int32_t* context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks,
                         float scale, pa_dtype dtype, pa_stream_t stream) {
    if (num_seqs > 0 && !slot_mapping) return fail(PA_ERR_INVALID_ARG, "null slot_mapping");
    return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       scale, dtype, key, value, slot_mapping, block_tables, stream);
}

size_t pa_decode_split_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                       int max_context_len, int partition_size) {
    if (num_seqs <= 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
        partition_size <= 0)
        return 0;
    const size_t parts = max_context_len == 0
                             ? 1
                             : (size_t)((max_context_len + (int64_t)partition_size - 1) /
                                        partition_size);
    const size_t heads = (size_t)num_seqs * num_heads;
    const size_t rows = heads * parts;
    size_t bytes = 2 * align256(rows * sizeof(float)) + align256(rows * head_dim * sizeof(float));
    const int chunks = reduce_chunks(heads, parts);
    if (chunks > 1)      // the reduce's per-chunk sums and arrival counts
        bytes += align256(heads * chunks * (head_dim + 4) * sizeof(float)) +
                 align256(heads * sizeof(unsigned));
    return bytes;
}

pa_status pa_decode_split(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_tables, int max_blocks_per_seq,
                          const int32_t* context_lens, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, int block_size, int num_blocks,
                          float scale, pa_dtype dtype, int max_context_len, int partition_size,
                          void* workspace, size_t workspace_bytes, pa_stream_t stream) {
    if (pa_status s = check_decode_args(out, q, k_cache, v_cache, block_tables,
                                        max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                        num_kv_heads, head_dim, block_size, num_blocks, dtype,
                                        scale))
        return s;
    if (partition_size <= 0 || partition_size % block_size != 0)
        return fail(PA_ERR_INVALID_ARG, "partition_size %d must be a positive multiple of %d",
                    partition_size, block_size);
    if (max_context_len < 0) return fail(PA_ERR_INVALID_ARG, "negative max_context_len");
    if (num_seqs == 0) return PA_OK;
    const size_t need = pa_decode_split_workspace_bytes(num_seqs, num_heads, head_dim,
                                                        max_context_len, partition_size);
    if (!workspace || workspace_bytes < need || !aligned16(workspace))
        return fail(PA_ERR_INVALID_ARG, "workspace needs %zu bytes, 16-byte aligned", need);
    const int64_t parts64 =
        max_context_len == 0 ? 1 : ((int64_t)max_context_len + partition_size - 1) / partition_size;
    if (parts64 > 0x7fffffff) return fail(PA_ERR_UNSUPPORTED, "too many partitions");
    if ((int64_t)num_seqs * num_heads > 0x7fffffff)
        return fail(PA_ERR_UNSUPPORTED, "num_seqs * num_heads overflows int32");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (validate_enabled())
        if (pa_status s = validate_decode(block_tables, max_blocks_per_seq, context_lens,
                                          num_seqs, block_size, num_blocks, st))
            return s;
    const size_t rows = (size_t)num_seqs * num_heads * (size_t)parts64;
    DecodeLaunch l = {};
    char* ws = static_cast<char*>(workspace);
    l.args.out = out;
    l.args.q = q;
    l.args.block_tables = block_tables;
    l.args.context_lens = context_lens;
    l.args.ws_m = reinterpret_cast<float*>(ws);
    l.args.ws_l = reinterpret_cast<float*>(ws + align256(rows * sizeof(float)));
    l.args.ws_o = reinterpret_cast<float*>(ws + 2 * align256(rows * sizeof(float)));
    const size_t heads = (size_t)num_seqs * num_heads;
    l.args.reduce_chunks = reduce_chunks(heads, (size_t)parts64);
    if (l.args.reduce_chunks > 1) {
        char* p = ws + 2 * align256(rows * sizeof(float)) +
                  align256(rows * head_dim * sizeof(float));
        l.args.ws_part = reinterpret_cast<float*>(p);
        l.args.ws_cnt = reinterpret_cast<unsigned*>(
            p + align256(heads * l.args.reduce_chunks * (head_dim + 4) * sizeof(float)));
    }
    if (pa_status s = set_error_and_waits(l.args)) return s;
    l.args.scale_log2 = scale * 1.4426950408889634f;
    l.args.num_seqs = num_seqs;
    l.args.max_blocks = max_blocks_per_seq;
    l.args.max_tokens = max_blocks_per_seq * block_size;
    l.args.num_heads = num_heads;
    l.args.num_kv_heads = num_kv_heads;
    l.args.num_blocks = num_blocks;
    l.args.part_tokens = partition_size;
    l.args.max_parts = (int)parts64;
    l.args.slot_stride = (int)parts64;
    l.k_cache = k_cache;
    l.v_cache = v_cache;
    l.num_seqs = num_seqs;
    l.num_kv_heads = num_kv_heads;
    l.block_size = block_size;
    l.group = num_heads / num_kv_heads;
    l.ctas = 1;
    l.split = true;
    l.stream = st;
    return dispatch_decode(l, dtype, head_dim);
}

size_t pa_decode_shared_prefix_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                               int max_prefix_len) {
    if (num_seqs <= 0 || num_heads <= 0 || head_dim <= 0 || max_prefix_len < 0) return 0;
    const int ct = prefix_chunk_tokens(head_dim);
    const size_t chunks = (size_t)((max_prefix_len + ct - 1) / ct);
    const size_t rows = (size_t)num_seqs * num_heads * (chunks ? chunks : 1);
    return 2 * align256(rows * sizeof(float)) + rows * head_dim * sizeof(float);
}

}  // extern "C"

namespace {

// pa_decode_shared_prefix, optionally as a whole step (new_slots and
// table_out both set): the own-token pass then also appends one new token
// per sequence (new_k/new_v at new_slots), taking each sequence's last block
// from its new slot and storing it in the table.
pa_status shared_prefix_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* context_lens, int num_seqs, int num_heads,
                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                             float scale, pa_dtype dtype, const int32_t* group_starts,
                             const int32_t* prefix_lens, int num_groups, int max_group_size,
                             int max_prefix_len, void* workspace, size_t workspace_bytes,
                             const void* new_k, const void* new_v, const int64_t* new_slots,
                             int32_t* table_out, pa_stream_t stream) {
    if (pa_status s = check_decode_args(out, q, k_cache, v_cache, block_tables,
                                        max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                        num_kv_heads, head_dim, block_size, num_blocks, dtype,
                                        scale))
        return s;
    if (dtype != PA_DTYPE_BF16)
        return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode needs bf16");
    if (num_groups <= 0 || max_group_size <= 0 || max_prefix_len < 0 ||
        (int64_t)max_prefix_len > (int64_t)max_blocks_per_seq * block_size)
        return fail(PA_ERR_INVALID_ARG, "bad group or prefix bounds");
    if ((int64_t)num_groups * ((max_group_size * (num_heads / num_kv_heads) +
                                PREFIX_ROWS_PER_CTA - 1) / PREFIX_ROWS_PER_CTA) > 65535)
        return fail(PA_ERR_UNSUPPORTED, "too many groups x row blocks for one launch");
    if (num_seqs == 0) return PA_OK;
    if (!group_starts || !prefix_lens) return fail(PA_ERR_INVALID_ARG, "null group arrays");
    const bool append = new_slots != nullptr;
    if (append && (!new_k || !new_v || !aligned16(new_k) || !aligned16(new_v)))
        return fail(PA_ERR_INVALID_ARG, "key and value rows must be 16-byte aligned device pointers");
    const size_t need = pa_decode_shared_prefix_workspace_bytes(num_seqs, num_heads, head_dim,
                                                                max_prefix_len);
    if (!workspace || workspace_bytes < need || !aligned16(workspace))
        return fail(PA_ERR_INVALID_ARG, "workspace needs %zu bytes, 16-byte aligned", need);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (validate_enabled()) {
        std::vector<int32_t> gs, pl, t, l;
        std::vector<int64_t> sl;
        if (!copy_to_host(gs, group_starts, (size_t)num_groups + 1, st) ||
            !copy_to_host(pl, prefix_lens, (size_t)num_groups, st) ||
            !copy_to_host(l, context_lens, (size_t)num_seqs, st) ||
            !copy_to_host(t, block_tables, (size_t)num_seqs * max_blocks_per_seq, st) ||
            (append && !copy_to_host(sl, new_slots, (size_t)num_seqs, st)))
            return fail(PA_ERR_CUDA, "validation copy failed");
        const int64_t num_slots = (int64_t)num_blocks * block_size;
        for (int s = 0; append && s < num_seqs; ++s) {
            // the new token: the sequence's last position, past its prefix
            // (checked below, per group), in the slot's row
            if (sl[s] < 0) continue;
            const int pos = l[s] - 1;
            if (sl[s] >= num_slots || pos < 0 ||
                (int64_t)pos >= (int64_t)max_blocks_per_seq * block_size)
                return fail(PA_ERR_BAD_BLOCK_ID, "new slot of sequence %d is %lld", s,
                            (long long)sl[s]);
            if (sl[s] % block_size != pos % block_size)
                return fail(PA_ERR_BAD_BLOCK_ID,
                            "new slot of sequence %d is %lld, not row %d of a pool block", s,
                            (long long)sl[s], pos % block_size);
            t[(size_t)s * max_blocks_per_seq + pos / block_size] = (int32_t)(sl[s] / block_size);
        }
        if (pa_status s = check_tables(t, l, max_blocks_per_seq, num_seqs, block_size, num_blocks))
            return s;
        if (gs[0] != 0 || gs[num_groups] != num_seqs)
            return fail(PA_ERR_BAD_BLOCK_ID, "groups must cover sequences 0..num_seqs-1");
        for (int g = 0; g < num_groups; ++g) {
            if (gs[g + 1] <= gs[g] || gs[g + 1] - gs[g] > max_group_size)
                return fail(PA_ERR_BAD_BLOCK_ID, "group %d is empty or above max_group_size", g);
            if (pl[g] < 0 || pl[g] > max_prefix_len || pl[g] % 16 || pl[g] % block_size)
                return fail(PA_ERR_BAD_BLOCK_ID, "prefix of group %d (%d) is not whole blocks "
                            "of 16 tokens within max_prefix_len", g, pl[g]);
            const int nb = pl[g] / block_size;
            for (int s = gs[g]; s < gs[g + 1]; ++s) {
                if (l[s] < pl[g])
                    return fail(PA_ERR_BAD_BLOCK_ID, "sequence %d is shorter than its prefix", s);
                if (append && sl[s] >= 0 && l[s] - 1 < pl[g])
                    return fail(PA_ERR_BAD_BLOCK_ID,
                                "the new token of sequence %d falls in its group's prefix", s);
                for (int j = 0; j < nb; ++j)
                    if (t[(size_t)s * max_blocks_per_seq + j] !=
                        t[(size_t)gs[g] * max_blocks_per_seq + j])
                        return fail(PA_ERR_BAD_BLOCK_ID,
                                    "sequence %d does not share block %d of its group's prefix",
                                    s, j);
            }
        }
    }
    const int chunk_tokens = prefix_chunk_tokens(head_dim);
    const int chunks = (max_prefix_len + chunk_tokens - 1) / chunk_tokens;
    const int group = num_heads / num_kv_heads;
    const size_t rows = (size_t)num_seqs * num_heads * (size_t)(chunks ? chunks : 1);
    char* ws = static_cast<char*>(workspace);
    DecodeLaunch l = {};
    l.args.out = out;
    l.args.q = q;
    l.args.block_tables = block_tables;
    l.args.context_lens = context_lens;
    l.args.ws_m = reinterpret_cast<float*>(ws);
    l.args.ws_l = reinterpret_cast<float*>(ws + align256(rows * sizeof(float)));
    l.args.ws_o = reinterpret_cast<float*>(ws + 2 * align256(rows * sizeof(float)));
    if (pa_status s = set_error_and_waits(l.args)) return s;
    l.args.scale_log2 = scale * 1.4426950408889634f;
    l.args.num_seqs = num_seqs;
    l.args.max_blocks = max_blocks_per_seq;
    l.args.max_tokens = max_blocks_per_seq * block_size;
    l.args.num_heads = num_heads;
    l.args.num_kv_heads = num_kv_heads;
    l.args.num_blocks = num_blocks;
    l.args.group_starts = group_starts;
    l.args.group_prefix = prefix_lens;
    l.args.num_groups = num_groups;
    l.args.chunk_tokens = chunk_tokens;
    l.args.prefix_slot0 = 0;
    l.args.slot_stride = chunks ? chunks : 1;
    l.args.sched = SCHED_LPT;
    l.args.new_k = new_k;
    l.args.new_v = new_v;
    l.args.new_slots = new_slots;
    l.args.table_out = table_out;
    l.args.k_cache = const_cast<void*>(k_cache);
    l.args.v_cache = const_cast<void*>(v_cache);
    l.k_cache = k_cache;
    l.v_cache = v_cache;
    l.num_seqs = num_seqs;
    l.num_kv_heads = num_kv_heads;
    l.block_size = block_size;
    l.group = group;
    l.ctas = 1;
    l.split = false;
    l.cascade = true;
    l.max_chunks = chunks;
    const int max_rows = max_group_size * group;
    l.row_blocks = (max_rows + PREFIX_ROWS_PER_CTA - 1) / PREFIX_ROWS_PER_CTA;
    l.stream = st;
    return dispatch_decode(l, dtype, head_dim);
}

}  // namespace

extern "C" {

pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  int max_blocks_per_seq, const int32_t* context_lens,
                                  int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                  int block_size, int num_blocks, float scale, pa_dtype dtype,
                                  const int32_t* group_starts, const int32_t* prefix_lens,
                                  int num_groups, int max_group_size, int max_prefix_len,
                                  void* workspace, size_t workspace_bytes, pa_stream_t stream) {
    return shared_prefix_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                              context_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                              block_size, num_blocks, scale, dtype, group_starts, prefix_lens,
                              num_groups, max_group_size, max_prefix_len, workspace,
                              workspace_bytes, nullptr, nullptr, nullptr, nullptr, stream);
}

pa_status pa_decode_shared_prefix_step(void* out, const void* q, const void* key,
                                       const void* value, void* k_cache, void* v_cache,
                                       const int64_t* slot_mapping, int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens,
                                       int num_seqs, int num_heads, int num_kv_heads,
                                       int head_dim, int block_size, int num_blocks, float scale,
                                       pa_dtype dtype, const int32_t* group_starts,
                                       const int32_t* prefix_lens, int num_groups,
                                       int max_group_size, int max_prefix_len, void* workspace,
                                       size_t workspace_bytes, pa_stream_t stream) {
    if (num_seqs > 0 && !slot_mapping) return fail(PA_ERR_INVALID_ARG, "null slot_mapping");
    return shared_prefix_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                              context_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                              block_size, num_blocks, scale, dtype, group_starts, prefix_lens,
                              num_groups, max_group_size, max_prefix_len, workspace,
                              workspace_bytes, key, value, slot_mapping, block_tables, stream);
}

pa_status pa_update_block_tables(int32_t* block_tables, int max_blocks_per_seq,
                                 const int32_t* context_lens, const int64_t* slot_mapping,
                                 int num_seqs, int block_size, int num_blocks,
                                 pa_stream_t stream) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || num_blocks <= 0)
        return fail(PA_ERR_INVALID_ARG, "sizes must be positive (num_seqs >= 0)");
    if (num_seqs == 0) return PA_OK;
    if (!block_tables || !context_lens || !slot_mapping)
        return fail(PA_ERR_INVALID_ARG, "null pointer");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (validate_enabled()) {
        std::vector<int32_t> l;
        std::vector<int64_t> sl;
        if (!copy_to_host(l, context_lens, (size_t)num_seqs, st) ||
            !copy_to_host(sl, slot_mapping, (size_t)num_seqs, st))
            return fail(PA_ERR_CUDA, "validation copy failed");
        for (int s = 0; s < num_seqs; ++s) {
            if (sl[s] < 0) continue;
            if (sl[s] >= (int64_t)num_blocks * block_size || l[s] <= 0 ||
                (l[s] - 1) / block_size >= max_blocks_per_seq)
                return fail(PA_ERR_BAD_BLOCK_ID, "sequence %d: slot %lld, length %d", s,
                            (long long)sl[s], l[s]);
            if (sl[s] % block_size != (l[s] - 1) % block_size)
                return fail(PA_ERR_BAD_BLOCK_ID,
                            "sequence %d: slot %lld is not at row %d of a block", s,
                            (long long)sl[s], (l[s] - 1) % block_size);
        }
    }
    return launch_update_tables(block_tables, max_blocks_per_seq, context_lens, slot_mapping,
                                num_seqs, block_size, num_blocks, st);
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                         int num_pairs, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, pa_dtype dtype, pa_stream_t stream) {
    if (num_pairs < 0 || num_kv_heads <= 0 || num_blocks <= 0)
        return fail(PA_ERR_INVALID_ARG, "sizes must be positive (num_pairs >= 0)");
    if (pa_status s = check_geometry(dtype, head_dim, block_size)) return s;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !block_mapping) return fail(PA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_INVALID_ARG, "caches must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (validate_enabled()) {
        std::vector<int64_t> mp;
        if (!copy_to_host(mp, block_mapping, (size_t)num_pairs * 2, st))
            return fail(PA_ERR_CUDA, "validation copy failed");
        std::unordered_set<int64_t> dsts, srcs;
        for (int i = 0; i < num_pairs; ++i) {
            for (int k = 0; k < 2; ++k)
                if (mp[2 * i + k] < 0 || mp[2 * i + k] >= num_blocks)
                    return fail(PA_ERR_BAD_BLOCK_ID, "block_mapping[%d] outside the pool", i);
            srcs.insert(mp[2 * i]);
            if (!dsts.insert(mp[2 * i + 1]).second)
                return fail(PA_ERR_BAD_BLOCK_ID, "destination %lld repeated",
                            (long long)mp[2 * i + 1]);
        }
        for (int64_t d : dsts)
            if (srcs.count(d))
                return fail(PA_ERR_BAD_BLOCK_ID, "block %lld is both source and destination",
                            (long long)d);
    }
    const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim * elem_size(dtype);
    return launch_copy_blocks(k_cache, v_cache, block_mapping, num_pairs, block_bytes, num_blocks,
                              st);
}

// Device-usable address of a pool: device or managed memory as is, pinned host
// memory through its device mapping; null if the GPU cannot reach it.
static void* device_view(const void* p) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();                       // pageable memory reports an error: clear it
        return nullptr;
    }
    if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged)
        return const_cast<void*>(p);
    if (attr.type == cudaMemoryTypeHost && attr.devicePointer) {
        // the mapping covers the whole allocation: offset the mapped base
        const uintptr_t off = reinterpret_cast<uintptr_t>(p) -
                              reinterpret_cast<uintptr_t>(attr.hostPointer);
        return static_cast<char*>(attr.devicePointer) + off;
    }
    return nullptr;
}

pa_status pa_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                         const int64_t* block_mapping, int num_pairs, int num_kv_heads,
                         int head_dim, int block_size, int src_num_blocks, int dst_num_blocks,
                         pa_dtype dtype, pa_stream_t stream) {
    if (num_pairs < 0 || num_kv_heads <= 0 || src_num_blocks <= 0 || dst_num_blocks <= 0)
        return fail(PA_ERR_INVALID_ARG, "sizes must be positive (num_pairs >= 0)");
    if (pa_status s = check_geometry(dtype, head_dim, block_size)) return s;
    if (num_pairs == 0) return PA_OK;
    if (!dst_k || !dst_v || !src_k || !src_v || !block_mapping)
        return fail(PA_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(dst_k) || !aligned16(dst_v) || !aligned16(src_k) || !aligned16(src_v))
        return fail(PA_ERR_INVALID_ARG, "pools must be 16-byte aligned");
    void* dk = device_view(dst_k);
    void* dv = device_view(dst_v);
    const void* sk = device_view(src_k);
    const void* sv = device_view(src_v);
    const void* mp = device_view(block_mapping);
    if (!dk || !dv || !sk || !sv || !mp)
        return fail(PA_ERR_UNSUPPORTED, "pools and mapping must be device memory or pinned "
                    "(device-mapped) host memory");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (validate_enabled()) {
        std::vector<int64_t> m;
        if (!copy_to_host(m, static_cast<const int64_t*>(mp), (size_t)num_pairs * 2, st))
            return fail(PA_ERR_CUDA, "validation copy failed");
        std::unordered_set<int64_t> dsts;
        for (int i = 0; i < num_pairs; ++i) {
            if (m[2 * i] < 0 || m[2 * i] >= src_num_blocks || m[2 * i + 1] < 0 ||
                m[2 * i + 1] >= dst_num_blocks)
                return fail(PA_ERR_BAD_BLOCK_ID, "block_mapping[%d] outside its pool", i);
            if (!dsts.insert(m[2 * i + 1]).second)
                return fail(PA_ERR_BAD_BLOCK_ID, "destination %lld repeated",
                            (long long)m[2 * i + 1]);
        }
    }
    const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim * elem_size(dtype);
    return launch_move_blocks(dk, dv, sk, sv, static_cast<const int64_t*>(mp), num_pairs,
                              block_bytes, src_num_blocks, dst_num_blocks, PA_DEVERR_COPY_ID, st);
}

}  // extern "C"
