// Internal helpers shared by the host-side translation units of
// libpagedattn.so (not part of the public ABI).
#pragma once

#include "pagedattn.h"

namespace pa {

// Record a printf-style message for pa_last_error() and return `status`.
pa_status fail(pa_status status, const char* fmt, ...)
#if defined(__GNUC__)
    __attribute__((format(printf, 2, 3)))
#endif
    ;

}  // namespace pa

#include <cuda.h>
#include <cuda_runtime.h>

namespace pa {

struct DecodeArgs;

// Encode a 4-D tensor map over a [num_blocks][block_size][kv_heads][head_dim]
// cache with a {box_inner, 1, rows, 1} box, optionally with the 128-byte
// shared-memory swizzle (box_inner * element size must then be 128 bytes).
pa_status encode_cache_map(CUtensorMap* map, const void* base, pa_dtype dtype, int head_dim,
                           int num_kv_heads, int block_size, int num_blocks, int box_inner,
                           int rows, bool swizzle128);

// Encode a 3-D tensor map over bf16 queries [num_seqs][num_heads][head_dim]
// with a {64, heads, seqs} box and the 128-byte swizzle: `heads` consecutive
// query heads of `seqs` consecutive sequences, one 128-byte row per (sequence,
// head), sequence-major.
pa_status encode_query_map(CUtensorMap* map, const void* q, int head_dim, int num_heads,
                           int num_seqs, int heads, int seqs);

// Device error word of the current device (address from cudaGetSymbolAddress).
unsigned* device_error_word();

// SM count of the current device.
int num_sms();

// PA_OPT_PDL: launch with programmatic stream serialisation.  Appends the
// attribute to attrs[*n] when enabled.
bool pdl_enabled();
void add_pdl_attr(cudaLaunchAttribute* attrs, unsigned* n);

// Everything a decode launch needs besides the template parameters.
struct DecodeLaunch;

pa_status launch_decode_f32_d64(const DecodeLaunch& l);
pa_status launch_decode_f32_d128(const DecodeLaunch& l);
pa_status launch_decode_f32_d256(const DecodeLaunch& l);
pa_status launch_decode_bf16_d64(const DecodeLaunch& l);
pa_status launch_decode_bf16_d128(const DecodeLaunch& l);
pa_status launch_decode_bf16_d256(const DecodeLaunch& l);

pa_status launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                   void* v_cache, const int64_t* slots, int num_tokens,
                                   int64_t row_bytes, int64_t num_slots, cudaStream_t stream);
pa_status launch_update_tables(int32_t* tables, int stride, const int32_t* lens,
                               const int64_t* slots, int num_seqs, int block_size,
                               int num_blocks, cudaStream_t stream);
pa_status launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* mapping, int num_pairs,
                             int64_t block_bytes, int num_blocks, cudaStream_t stream);
pa_status launch_move_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                             const int64_t* mapping, int num_pairs, int64_t block_bytes,
                             int src_blocks, int dst_blocks, unsigned err_bits,
                             cudaStream_t stream);

}  // namespace pa
