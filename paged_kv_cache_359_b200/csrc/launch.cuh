// Host-side launch of the paged decode kernels for one (dtype, head_dim);
// dispatches block_size and group size to template instances.
#pragma once

#include <atomic>
#include <type_traits>

#include "decode.cuh"
#include "internal.h"
#include "prefix.cuh"

namespace pa {

struct DecodeLaunch {
    DecodeArgs args;
    const void* k_cache;
    const void* v_cache;
    int num_seqs;
    int num_kv_heads;
    int block_size;
    int group;
    int ctas;          // pa_decode: CTAs (one cluster) per (sequence, kv head)
    bool split;
    // shared-prefix decode: the shared pass runs first (grid max_chunks x Hk x
    // groups * row_blocks), then pa_decode's kernel over the own tokens
    bool cascade;
    int max_chunks;
    int row_blocks;
    cudaStream_t stream;
};

// Opt a kernel into `bytes` of dynamic shared memory, once per device, and
// prefer all of L1 as shared memory: the decode kernels fill an SM's shared
// memory anyway, and the cascade's two kernels can then share an SM (a
// decode CTA beside a shared-pass CTA).  `done` must be distinct for every
// kernel (one static per instantiation).
template <class K>
inline pa_status allow_smem(K kernel, int bytes, std::atomic<unsigned long long>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice failed");
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_relaxed) & bit) return PA_OK;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess)
        return fail(PA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    done.fetch_or(bit);
    return PA_OK;
}

template <typename T, int D, int BS, int G>
pa_status launch_decode_g(const DecodeLaunch& l) {
    using U = UnitFor<T, D, BS, G>;
    using Ly = Layout<U>;
    constexpr pa_dtype DT = std::is_same<T, float>::value ? PA_DTYPE_F32 : PA_DTYPE_BF16;
    CUtensorMap mk, mv;
    if (pa_status s = encode_cache_map(&mk, l.k_cache, DT, D, l.num_kv_heads, BS,
                                       l.args.num_blocks, U::BOX_INNER, U::BOX_ROWS,
                                       U::SWIZZLE128))
        return s;
    if (pa_status s = encode_cache_map(&mv, l.v_cache, DT, D, l.num_kv_heads, BS,
                                       l.args.num_blocks, U::BOX_INNER, U::BOX_ROWS,
                                       U::SWIZZLE128))
        return s;
    if (l.split && l.args.part_tokens % U::R != 0)
        return fail(PA_ERR_INVALID_ARG, "partition must be a multiple of %d tokens", U::R);

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    cfg.attrs = attr;
    add_pdl_attr(attr, &cfg.numAttrs);
    cfg.blockDim = dim3(Ly::NW * 32);
    cfg.dynamicSmemBytes = Ly::SMEM_BYTES;
    cfg.stream = l.stream;
    cudaError_t e;
    if (l.cascade) {
        if constexpr (std::is_same<T, __nv_bfloat16>::value && (BS % 16 == 0 || BS == 8)) {
            using C = PrefixCfg<D, BS, G>;
            static std::atomic<unsigned long long> done_p{0};
            auto pk = shared_prefix_kernel<D, BS, G>;
            if (pa_status s = allow_smem(pk, C::SMEM_BYTES, done_p)) return s;
            CUtensorMap sq, sk, sv;    // 128B-swizzled boxes: q {64, G, 128 / G}, K/V {64, 1, 16 or 8, 1}
            if (pa_status s = encode_query_map(&sq, l.args.q, D, l.args.num_heads, l.num_seqs,
                                               G, C::M / G))
                return s;
            if (pa_status s = encode_cache_map(&sk, l.k_cache, DT, D, l.num_kv_heads, BS,
                                               l.args.num_blocks, 64, C::BOX_ROWS, true))
                return s;
            if (pa_status s = encode_cache_map(&sv, l.v_cache, DT, D, l.num_kv_heads, BS,
                                               l.args.num_blocks, 64, C::BOX_ROWS, true))
                return s;
            if (l.max_chunks > 0) {
                cudaLaunchConfig_t pc = {};
                pc.gridDim = dim3(l.max_chunks, l.num_kv_heads, l.args.num_groups * l.row_blocks);
                pc.blockDim = dim3(C::THREADS);
                pc.dynamicSmemBytes = C::SMEM_BYTES;
                pc.stream = l.stream;
                cudaLaunchAttribute pattr[1];
                pc.attrs = pattr;
                add_pdl_attr(pattr, &pc.numAttrs);
                e = cudaLaunchKernelEx(&pc, pk, sq, sk, sv, l.args, l.row_blocks);
                if (e != cudaSuccess)
                    return fail(PA_ERR_CUDA, "shared-prefix launch: %s", cudaGetErrorString(e));
            }
            // the own-token pass: longest-first (half-width CTAs but at head_dim 256)
            using Lo = Layout<U, own_half_width<U>()>;
            static std::atomic<unsigned long long> done_o{0};
            auto ok = paged_decode_kernel<U, Mode::Own>;
            if (pa_status s = allow_smem(ok, Lo::SMEM_BYTES, done_o)) return s;
            cfg.blockDim = dim3(Lo::NW * 32);
            cfg.dynamicSmemBytes = Lo::SMEM_BYTES;
            cfg.gridDim = dim3((unsigned)((long long)l.num_seqs * l.num_kv_heads));
            // The own-token pass reads the cache before its dependency wait,
            // which is safe only behind the shared pass (whose CTAs wait for
            // the stream's previous kernel before they release it).  Without
            // a shared pass it launches in plain stream order.
            if (l.max_chunks <= 0) cfg.numAttrs = 0;
            e = cudaLaunchKernelEx(&cfg, ok, mk, mv, l.args);
            if (e != cudaSuccess)
                return fail(PA_ERR_CUDA, "own-token launch: %s", cudaGetErrorString(e));
            return PA_OK;
        } else {
            return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode needs bf16");
        }
    }
    if (l.split) {
        static std::atomic<unsigned long long> done{0};
        auto kern = paged_decode_kernel<U, Mode::Split>;
        if (pa_status s = allow_smem(kern, Ly::SMEM_BYTES, done)) return s;
        cfg.gridDim = dim3(l.args.max_parts, l.num_kv_heads, l.num_seqs);
        e = cudaLaunchKernelEx(&cfg, kern, mk, mv, l.args);
        if (e == cudaSuccess) {
            cudaLaunchConfig_t rc = {};
            rc.gridDim = dim3(l.num_seqs * l.args.num_heads, l.args.reduce_chunks);
            rc.blockDim = dim3(256);
            rc.stream = l.stream;
            cudaLaunchAttribute rattr[1];
            rc.attrs = rattr;
            add_pdl_attr(rattr, &rc.numAttrs);
            e = cudaLaunchKernelEx(&rc, lse_reduce_kernel<T, D>, l.args);
        }
    } else if (l.args.sched == SCHED_LPT) {
        static std::atomic<unsigned long long> done{0};
        auto kern = paged_decode_kernel<U, Mode::Decode>;
        if (pa_status s = allow_smem(kern, Ly::SMEM_BYTES, done)) return s;
        cfg.gridDim = dim3((unsigned)((long long)l.num_seqs * l.num_kv_heads));
        e = cudaLaunchKernelEx(&cfg, kern, mk, mv, l.args);
    } else {
        static std::atomic<unsigned long long> done{0};
        auto kern = paged_decode_kernel<U, Mode::Cluster>;
        if (pa_status s = allow_smem(kern, Ly::SMEM_BYTES, done)) return s;
        cfg.gridDim = dim3(l.ctas, l.num_kv_heads, l.num_seqs);
        if (l.ctas > 1) {
            cudaLaunchAttribute& c = attr[cfg.numAttrs++];
            c.id = cudaLaunchAttributeClusterDimension;
            c.val.clusterDim.x = l.ctas;
            c.val.clusterDim.y = 1;
            c.val.clusterDim.z = 1;
        }
        e = cudaLaunchKernelEx(&cfg, kern, mk, mv, l.args);
    }
    if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return PA_OK;
}

template <typename T, int D, int BS>
pa_status launch_decode_bs(const DecodeLaunch& l) {
    switch (l.group) {
        case 1: return launch_decode_g<T, D, BS, 1>(l);
        case 2: return launch_decode_g<T, D, BS, 2>(l);
        case 4: return launch_decode_g<T, D, BS, 4>(l);
        case 8: return launch_decode_g<T, D, BS, 8>(l);
        default: return fail(PA_ERR_UNSUPPORTED, "group size %d not built", l.group);
    }
}

template <typename T, int D>
pa_status launch_decode_td(const DecodeLaunch& l) {
    switch (l.block_size) {
        case 8: return launch_decode_bs<T, D, 8>(l);
        case 16: return launch_decode_bs<T, D, 16>(l);
        case 32: return launch_decode_bs<T, D, 32>(l);
        case 64: return launch_decode_bs<T, D, 64>(l);
        case 128: return launch_decode_bs<T, D, 128>(l);
        default: return fail(PA_ERR_UNSUPPORTED, "block_size %d not built", l.block_size);
    }
}

}  // namespace pa

#define PA_DEFINE_DECODE_LAUNCHER(NAME, T, D) \
    namespace pa {                            \
    pa_status NAME(const DecodeLaunch& l) { return launch_decode_td<T, D>(l); } \
    }
