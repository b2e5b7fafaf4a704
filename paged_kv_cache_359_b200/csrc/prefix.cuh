// Shared-prefix pass of the cascade decode (sm_100a, bf16).
//
// Sequences forked from one prompt share its blocks ("vLLM内存管理与
// PagedAttention精讲" ch.2 §2.4.3: several requests' block tables point at
// the same physical blocks; "VLLM中PagedAttention如何降低显存碎片？" §三
// item 8: shared prefix pages).  Plain decode re-reads those blocks once per
// sharer.  Here the members of a group attend over the shared prefix
// together: the query rows of all members (members x G heads of one kv
// head) form the M side of a real dense contraction, so each prefix tile is
// read from HBM once per kv head (the row blocks of one chunk run together
// and share it through L2) instead of once per sequence.
//
// CTA = (prefix chunk of 256 tokens, kv head, group x 64-row block).  One
// producer warp streams the chunk's 16-token units with TMA into a ring of
// STAGES shared-memory stages (full / empty mbarriers, bounded waits); up to
// 4 consumer warps each own 16 query rows (two CTAs fit an SM) and run
//   S[16 x 16] = Q K^T,  O[16 x D] += P V
// with mma.sync m16n8k16 (bf16 in, fp32 accumulate), an online softmax with
// a lazy running max, and write the chunk's (max, sum, unnormalised output)
// per row to the workspace slot prefix_slot0 + chunk; pa_decode's CTAs for
// each sequence's own tokens merge them into the output.
#pragma once

#include "decode.cuh"

namespace pa {

template <int D_, int BS_, int G_>
struct PrefixCfg {
    static constexpr int D = D_, BS = BS_, G = G_;
    static constexpr int R = 16;                 // tokens per unit
    // 8-token blocks: a unit's rows 0..7 and 8..15 are two 8-row boxes from
    // consecutive table entries, the second one swizzle atom further on
    static constexpr int BOX_ROWS = BS < R ? BS : R;
    static constexpr int BOXES = D / 64;         // 128-byte swizzled boxes per tile
    static constexpr int BOX_BYTES = R * 128;
    static constexpr int KS = D / 16, NT = D / 8;
    static constexpr int STAGE_BYTES = 2 * R * D * 2;
    static constexpr int STAGES = D >= 256 ? 4 : 8;
    static constexpr int MAX_CONSUMERS = 4;      // 64 query rows per CTA: two CTAs per SM
    static constexpr int THREADS = (MAX_CONSUMERS + 1) * 32;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 2 * STAGES * 8 + 1024;
    static_assert((BS % R == 0 || BS == 8) && D % 64 == 0, "shared-prefix shape");
};

constexpr int PREFIX_CHUNK_TOKENS = 256;
constexpr int PREFIX_ROWS_PER_CTA = 64;

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// byte offset of 16-byte chunk `chunk` (of D/8) in row `row` of a swizzled tile
__device__ __forceinline__ uint32_t swz128(int row, int chunk) {
    return (uint32_t)((chunk >> 3) * (16 * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

template <int D, int BS, int G>
__global__ void __launch_bounds__(PrefixCfg<D, BS, G>::THREADS)
    shared_prefix_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a,
                         int row_blocks) {
    pdl_wait();
    pdl_launch_dependents();
    using C = PrefixCfg<D, BS, G>;
    constexpr int R = C::R, STAGES = C::STAGES, KS = C::KS, NT = C::NT;
    const int chunk = blockIdx.x, kvh = blockIdx.y;
    const int grp = blockIdx.z / row_blocks, rblk = blockIdx.z % row_blocks;
    const int gs = __ldg(a.group_starts + grp), ge = __ldg(a.group_starts + grp + 1);
    const int prefix = __ldg(a.group_prefix + grp);
    const int rows = (ge - gs) * G;
    const int row0 = rblk * PREFIX_ROWS_PER_CTA;
    const int nunits = prefix / R;
    const int u_begin = chunk * (a.chunk_tokens / R);
    const int u_end = cmin(u_begin + a.chunk_tokens / R, nunits);
    if (u_begin >= u_end || row0 >= rows) return;     // whole CTA, before any barrier
    const int nk = u_end - u_begin;
    const int consumers = (blockDim.x / 32) - 1;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], consumers);
        }
        fence_mbar_init();
    }
    __syncthreads();
    // the members share their first prefix / BS table entries: read the first member's
    const int32_t* table = a.block_tables + (size_t)gs * a.max_blocks;

    if (warp == consumers) {
        // ---------------- producer warp: lane 0 streams the chunk's units ----------------
        if (lane == 0) {
            for (int k = 0; k < nk; ++k) {
                const int s = k % STAGES;
                if (k >= STAGES &&
                    !mbar_wait_bounded(&empty[s], ((k / STAGES) - 1) & 1, a.wait_ns)) {
                    raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
                    break;                  // consumers time out on `full` and finish
                }
                const int u = u_begin + k;
                auto checked = [&](int id) {
                    if (id < 0 || id >= a.num_blocks) {
                        raise_error(a.err, PA_DEVERR_BLOCK_ID);
                        return a.num_blocks;
                    }
                    return id;
                };
                // the prefix is whole 16-token units, so both halves of a unit exist
                const int id = checked(__ldg(table + (u * R) / BS));
                const int id1 = C::BOX_ROWS < R ? checked(__ldg(table + (u * R) / BS + 1)) : id;
                const int rr = C::BOX_ROWS < R ? 0 : (u * R) % BS;
                unsigned char* kdst = smem + s * C::STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES + a.tx_extra);
#pragma unroll
                for (int b = 0; b < C::BOXES; ++b) {
                    unsigned char* kb = kdst + b * C::BOX_BYTES;
                    unsigned char* vb = kb + C::STAGE_BYTES / 2;
                    tma_load_4d(kb, &tm_k, &full[s], b * 64, kvh, rr, id);
                    tma_load_4d(vb, &tm_v, &full[s], b * 64, kvh, rr, id);
                    if (C::BOX_ROWS < R) {
                        constexpr int OFF = C::BOX_ROWS * 128;     // bytes
                        tma_load_4d(kb + OFF, &tm_k, &full[s], b * 64, kvh, 0, id1);
                        tma_load_4d(vb + OFF, &tm_v, &full[s], b * 64, kvh, 0, id1);
                    }
                }
            }
        }
        return;
    }

    // ---------------- consumer warps: 16 query rows each ----------------
    // rows r0 = lane/4 and r1 = r0 + 8 of this warp's tile; row r -> member r / G, head r % G
    const int wrow = row0 + 16 * warp;
    const int r0 = wrow + (lane >> 2), r1 = r0 + 8;
    const int c2 = 2 * (lane & 3);
    const bool v0 = r0 < rows, v1 = r1 < rows;
    auto qrow = [&](int r) {
        const int seq = gs + r / G, h = kvh * G + r % G;
        return reinterpret_cast<const uint32_t*>(reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                                 ((size_t)seq * a.num_heads + h) * D);
    };
    uint32_t qa[KS][4];
    {
        const uint32_t* q0 = v0 ? qrow(r0) : nullptr;
        const uint32_t* q1 = v1 ? qrow(r1) : nullptr;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            qa[k][0] = v0 ? __ldg(q0 + (16 * k + c2) / 2) : 0u;
            qa[k][1] = v1 ? __ldg(q1 + (16 * k + c2) / 2) : 0u;
            qa[k][2] = v0 ? __ldg(q0 + (16 * k + 8 + c2) / 2) : 0u;
            qa[k][3] = v1 ? __ldg(q1 + (16 * k + 8 + c2) / 2) : 0u;
        }
    }
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    const int mi = lane >> 3, rr = lane & 7;
    bool failed = false;
    for (int k = 0; k < nk; ++k) {
        const int s = k % STAGES;
        if (!__all_sync(FULL_MASK, mbar_wait_bounded(&full[s], (k / STAGES) & 1, a.wait_ns))) {
            if (lane == 0) raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
            // later stages the producer may have issued: bounded waits
            for (int kk = k + 1; kk < cmin(nk, k + STAGES); ++kk)
                (void)mbar_wait_bounded(&full[kk % STAGES], (kk / STAGES) & 1, a.wait_ns);
            failed = true;
            break;
        }
        const uint32_t kb = smem_addr(smem + s * C::STAGE_BYTES);
        const uint32_t vb = kb + C::STAGE_BYTES / 2;
        // S = Q K^T for 16 rows x 16 tokens
        // two accumulators per n-tile (even / odd k-steps) halve the dependent chain
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        {
            float t0[4] = {0.f, 0.f, 0.f, 0.f}, t1[4] = {0.f, 0.f, 0.f, 0.f};
            const int tok = 8 * (mi >> 1) + rr;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t b[4];
                ldmatrix_x4(b, kb + swz128(tok, 2 * kk + (mi & 1)));
                float(&u0)[4] = (kk & 1) ? t0 : s0;
                float(&u1)[4] = (kk & 1) ? t1 : s1;
                mma_bf16_16816(u0, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b[0], b[1]);
                mma_bf16_16816(u1, qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                s0[j] += t0[j];
                s1[j] += t1[j];
            }
        }
        // rows r0: s0[0..1], s1[0..1]; rows r1: s0[2..3], s1[2..3] (log2 units)
        float x0[4] = {s0[0] * a.scale_log2, s0[1] * a.scale_log2, s1[0] * a.scale_log2,
                       s1[1] * a.scale_log2};
        float x1[4] = {s0[2] * a.scale_log2, s0[3] * a.scale_log2, s1[2] * a.scale_log2,
                       s1[3] * a.scale_log2};
        const float mx0 = fmaxf(fmaxf(x0[0], x0[1]), fmaxf(x0[2], x0[3]));
        const float mx1 = fmaxf(fmaxf(x1[0], x1[1]), fmaxf(x1[2], x1[3]));
        if (__any_sync(FULL_MASK, mx0 > m0 + RESCALE_THRESHOLD || mx1 > m1 + RESCALE_THRESHOLD)) {
            float a0 = mx0, a1 = mx1;
            a0 = fmaxf(a0, __shfl_xor_sync(FULL_MASK, a0, 1));
            a0 = fmaxf(a0, __shfl_xor_sync(FULL_MASK, a0, 2));
            a1 = fmaxf(a1, __shfl_xor_sync(FULL_MASK, a1, 1));
            a1 = fmaxf(a1, __shfl_xor_sync(FULL_MASK, a1, 2));
            const float n0 = fmaxf(m0, a0), n1 = fmaxf(m1, a1);
            const float al0 = exp2_approx(m0 - n0), al1 = exp2_approx(m1 - n1);
            m0 = n0;
            m1 = n1;
            l0 *= al0;
            l1 *= al1;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                o[n][0] *= al0;
                o[n][1] *= al0;
                o[n][2] *= al1;
                o[n][3] *= al1;
            }
        }
        float p0[4], p1[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            p0[j] = exp2_approx(x0[j] - m0);
            p1[j] = exp2_approx(x1[j] - m1);
            l0 += p0[j];
            l1 += p1[j];
        }
        const uint32_t pa0 = pack_bf16x2(p0[0], p0[1]), pa1 = pack_bf16x2(p1[0], p1[1]);
        const uint32_t pa2 = pack_bf16x2(p0[2], p0[3]), pa3 = pack_bf16x2(p1[2], p1[3]);
        // O += P V
        {
            const int tok = 8 * (mi & 1) + rr;
#pragma unroll
            for (int j = 0; j < NT / 2; ++j) {
                uint32_t b[4];
                ldmatrix_x4_trans(b, vb + swz128(tok, 2 * j + (mi >> 1)));
                mma_bf16_16816(o[2 * j], pa0, pa1, pa2, pa3, b[0], b[1]);
                mma_bf16_16816(o[2 * j + 1], pa0, pa1, pa2, pa3, b[2], b[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (failed) {
        // the error word says so; wait (bounded) for stages the producer may
        // still have in flight, then leave without writing anything
        return;
    }
    l0 += __shfl_xor_sync(FULL_MASK, l0, 1);
    l0 += __shfl_xor_sync(FULL_MASK, l0, 2);
    l1 += __shfl_xor_sync(FULL_MASK, l1, 1);
    l1 += __shfl_xor_sync(FULL_MASK, l1, 2);
    const int slot_in = a.prefix_slot0 + chunk;
    auto write_row = [&](int r, float mm, float ll, int half) {
        const int seq = gs + r / G, h = kvh * G + r % G;
        const size_t slot = ((size_t)seq * a.num_heads + h) * a.slot_stride + slot_in;
        if ((lane & 3) == 0) {
            a.ws_m[slot] = mm;
            a.ws_l[slot] = ll;
        }
        float* dst = a.ws_o + slot * D + c2;
#pragma unroll
        for (int n = 0; n < NT; ++n)
            *reinterpret_cast<float2*>(dst + 8 * n) = make_float2(o[n][2 * half], o[n][2 * half + 1]);
    };
    if (v0) write_row(r0, m0, l0, 0);
    if (v1) write_row(r1, m1, l1, 1);
}

}  // namespace pa
