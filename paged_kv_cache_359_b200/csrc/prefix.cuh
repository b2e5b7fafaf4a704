// Shared-prefix pass of the cascade decode on the 5th-generation tensor
// cores (sm_100a, bf16).
//
// Sequences forked from one prompt share its blocks ("vLLM内存管理与
// PagedAttention精讲" ch.2 §2.4.3: several requests' block tables point at
// the same physical blocks; "VLLM中PagedAttention如何降低显存碎片？" §三
// item 8: shared prefix pages).  Plain decode re-reads those blocks once per
// sharer.  Here the members of a group attend over the shared prefix
// together: the query rows of all members (members x G heads of one kv
// head) form the M side of a dense contraction, so each prefix tile is read
// from HBM once per kv head (once per 128 query rows from L2) instead of
// once per sequence.
//
// CTA = (prefix chunk of CH tokens, kv head, group x 128-row block); CH is
// 256 (head_dim <= 128) or 128 (head_dim 256).  Roles:
//  * producer warp: TMA loads of the CTA's 128 query rows (a 3-D box over
//    q [S][Hq][D]: members x G heads, row = member * G + head) and of the
//    chunk's K tiles in groups of 64 tokens, all 128-byte swizzled; once the
//    first MMA has read Q, the chunk's V tiles into Q's space (so the CTA
//    needs ~128 KB of shared memory and a decode CTA fits beside it); a
//    unit past the prefix is loaded from outside the pool map, which TMA
//    fills with zeros;
//  * MMA warp (one elected thread): S = Q K^T into TMEM (M = 128 rows,
//    N = 64 tokens per group as its K tiles land, K = head_dim), commit;
//    then, once P is in shared memory, O = P V into TMEM (M = 128,
//    N = head_dim, K = CH tokens, V read MN-major), commit;
//  * four softmax warps, one TMEM lane (query row) per thread: the exact
//    maximum of the row's scores over the chunk (masked past the prefix),
//    then p = 2^(s * scale * log2 e - max), rounded to bf16, into the
//    swizzled P tile (which reuses the K tile's space) and the fp32 sum of p;
//    after the second MMA each thread stages its row's output in the (now
//    free) tiles, up to 128 columns at a time, and sends it with one TMA
//    bulk copy to the workspace slot prefix_slot0 + chunk, with the row's
//    maximum and sum; pa_decode's CTAs for each sequence's own tokens merge
//    these into the output.
// Every wait is bounded; a wait that runs out sets PA_DEVERR_WAIT_TIMEOUT,
// the CTA skips what depends on it, waits (bounded) for its own loads and
// MMAs, frees its TMEM and leaves without writing.
#pragma once

#include "decode.cuh"

namespace pa {

template <int D_, int BS_, int G_>
struct PrefixCfg {
    static constexpr int D = D_, BS = BS_, G = G_;
    static constexpr int R = 16;                       // tokens per unit (one or two TMA boxes)
    static constexpr int BOX_ROWS = BS < R ? BS : R;   // 8-token blocks: two boxes per unit
    static constexpr int CH = D <= 128 ? 256 : 128;    // chunk tokens
    static constexpr int U = CH / R;                   // units per chunk
    static constexpr int NG = CH / 64;                 // 64-token groups (S MMAs, K barriers)
    static constexpr int KSL = D / 64;                 // 64-dim slabs of a 128-byte-swizzled tile
    static constexpr int M = 128;                      // query rows per CTA
    static constexpr int Q_BYTES = KSL * M * 128;
    static constexpr int KV_BYTES = KSL * CH * 128;
    static constexpr int P_BYTES = NG * M * 128;
    static constexpr int KP_BYTES = KV_BYTES > P_BYTES ? KV_BYTES : P_BYTES;
    static constexpr int QV_BYTES = KV_BYTES > Q_BYTES ? KV_BYTES : Q_BYTES;
    // Q, then V over the same bytes; K, then P over the same bytes
    static constexpr int QV_OFF = 0, K_OFF = QV_BYTES;
    static constexpr int BAR_OFF = QV_BYTES + KP_BYTES;
    // q_full, k_full[NG], v_full, s_full[NG], p_full, o_full; then the TMEM address
    static constexpr int NBARS = 2 * NG + 4;
    static constexpr int SOFT_WARPS = 4;
    static constexpr int PRODUCER = SOFT_WARPS, MMA_WARP = SOFT_WARPS + 1;
    static constexpr int THREADS = (SOFT_WARPS + 2) * 32;
    // the output is staged OCOLS columns at a time, rows padded by 4 floats
    static constexpr int OCOLS = D < 128 ? D : 128;
    static constexpr int OSTRIDE = OCOLS + 4;
    // barriers, the TMEM address, agreement flags, then alignment slack
    static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 16 + 2 * 4 * 4 + 1024;
    static constexpr int TMEM_COLS = 512;             // S at column 0, O at column CH
    static_assert(M * OSTRIDE * 4 <= BAR_OFF, "staged output fits the freed tiles");
    static_assert((BS % R == 0 || BS == 8) && D % 64 == 0, "shared-prefix shape");
    static_assert(CH + D <= TMEM_COLS, "S and O must fit TMEM");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

constexpr int PREFIX_ROWS_PER_CTA = 128;

// Tokens per prefix chunk (one CTA's share of the shared prefix).
__host__ __device__ constexpr int prefix_chunk_tokens(int head_dim) {
    return head_dim <= 128 ? 256 : 128;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

template <int D, int BS, int G>
__global__ void __launch_bounds__(PrefixCfg<D, BS, G>::THREADS, 1)
    shared_prefix_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a,
                         int row_blocks) {
    using C = PrefixCfg<D, BS, G>;
    constexpr int R = C::R, CH = C::CH, NG = C::NG, KSL = C::KSL, M = C::M;
    pdl_wait();
    pdl_launch_dependents();
    const int chunk = blockIdx.x, kvh = blockIdx.y;
    const int grp = blockIdx.z / row_blocks, rblk = blockIdx.z % row_blocks;
    const int gs = __ldg(a.group_starts + grp), ge = __ldg(a.group_starts + grp + 1);
    const int prefix = __ldg(a.group_prefix + grp);
    const int rows = (ge - gs) * G;
    const int row0 = rblk * M;
    const int nunits = prefix / R;
    const int u_begin = chunk * C::U;
    const int u_end = cmin(u_begin + C::U, nunits);
    if (u_begin >= u_end || row0 >= rows) return;       // whole CTA, before any barrier
    const int valid = (u_end - u_begin) * R;             // tokens of this chunk in the prefix
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* qs = smem + C::QV_OFF;                 // Q, then V
    unsigned char* ks = smem + C::K_OFF;                  // K tiles, then P
    unsigned char* vs = qs;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;                          // [NG]
    uint64_t* v_full = bars + 1 + NG;
    uint64_t* s_full = v_full + 1;                        // [NG]: S of 64-token group g done
    uint64_t* p_full = s_full + NG;
    uint64_t* o_full = p_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
    int* okw = reinterpret_cast<int*>(tmem_slot + 4);             // [2][SOFT_WARPS]
    // set by a role that gave up, read by the others after the final barrier
    __shared__ int failed;

    if (threadIdx.x == 0) {
        failed = 0;
        for (int i = 0; i < C::NBARS; ++i)
            mbar_init(&bars[i], i == 2 * NG + 2 ? 32 * C::SOFT_WARPS : 1);
        fence_mbar_init();
    }
    if (warp == C::MMA_WARP) {                            // the MMA warp owns TMEM
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t s_tmem = tmem, o_tmem = tmem + CH;
    bool v_issued = false;                                // producer lane 0 only

    if (warp == C::PRODUCER) {
        // ------------------------------------------------ producer (lane 0) --
        if (lane == 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            // the members share their first prefix / BS table entries: read the first member's
            const int32_t* table = a.block_tables + (size_t)gs * a.max_blocks;
            auto checked = [&](int id) {
                if (id < 0 || id >= a.num_blocks) {
                    raise_error(a.err, PA_DEVERR_BLOCK_ID);
                    return a.num_blocks;          // outside the map: TMA fills zeros
                }
                return id;
            };
            mbar_arrive_expect_tx(q_full, C::Q_BYTES + a.tx_extra);
#pragma unroll
            for (int b = 0; b < KSL; ++b)
                tma_load_3d(qs + b * M * 128, &tm_q, q_full, 64 * b, kvh * G, gs + row0 / G);
            // unit j of the chunk lands at row 16 j of every 64-dim slab
            auto load_unit = [&](const CUtensorMap* map, unsigned char* base, uint64_t* bar,
                                 int j) {
                const int u = u_begin + j;
                int id = a.num_blocks, id1 = a.num_blocks, rr = 0;
                if (u < u_end) {                    // the prefix is whole 16-token units
                    id = checked(__ldg(table + (u * R) / BS));
                    if (C::BOX_ROWS < R) id1 = checked(__ldg(table + (u * R) / BS + 1));
                    else rr = (u * R) % BS;
                }
#pragma unroll
                for (int b = 0; b < KSL; ++b) {
                    unsigned char* dst = base + b * CH * 128 + j * R * 128;
                    tma_load_4d(dst, map, bar, 64 * b, kvh, rr, id);
                    if (C::BOX_ROWS < R)
                        tma_load_4d(dst + C::BOX_ROWS * 128, map, bar, 64 * b, kvh, 0, id1);
                }
            };
            for (int g = 0; g < NG; ++g) {
                mbar_arrive_expect_tx(&k_full[g], 4 * KSL * R * 128 + a.tx_extra);
                for (int j = 4 * g; j < 4 * g + 4; ++j) load_unit(&tm_k, ks, &k_full[g], j);
            }
            // V goes over Q once the first MMA has read it (the last group's
            // commit covers every S MMA)
            if (mbar_wait_bounded(&s_full[NG - 1], 0, a.wait_ns)) {
                mbar_arrive_expect_tx(v_full, C::KV_BYTES + a.tx_extra);
                for (int j = 0; j < C::U; ++j) load_unit(&tm_v, vs, v_full, j);
                v_issued = true;
            } else {
                raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
                failed = 1;
            }
        }
    } else if (warp == C::MMA_WARP) {
        // --------------------------------------------- MMA issuer (lane 0) --
        if (lane == 0) {
            const uint32_t q0 = smem_addr(qs), k0 = smem_addr(ks), v0 = smem_addr(vs);
            // base descriptors; a step's operand is the base plus a byte
            // offset (>> 4) added to the start-address field, which stays
            // inside its 14 bits for any shared-memory address
            const uint64_t qd = sw128_desc(q0, 16, 1024), kd = sw128_desc(k0, 16, 1024);
            const uint64_t pd = kd, vd = sw128_desc(v0, CH * 128, 1024);
            bool ok = mbar_wait_bounded(q_full, 0, a.wait_ns);
            bool s_issued = false;
            if (ok) {
                for (int g = 0; g < NG && ok; ++g) {
                    ok = mbar_wait_bounded(&k_full[g], 0, a.wait_ns);
                    if (!ok) break;
                    tc_fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < 4 * KSL; ++kk) {
                        const uint64_t ad = qd + (uint64_t)(((kk / 4) * M * 128 + (kk % 4) * 32) >> 4);
                        const uint64_t bd =
                            kd + (uint64_t)(((kk / 4) * CH * 128 + g * 64 * 128 + (kk % 4) * 32) >> 4);
                        umma_bf16(s_tmem + 64 * g, ad, bd, umma_idesc_bf16(M, 64, false),
                                  kk > 0);
                    }
                    umma_commit(&s_full[g]);          // the softmax starts on this group
                    s_issued = true;
                }
            }
            bool o_issued = false;
            if (ok) ok = mbar_wait_bounded(p_full, 0, a.wait_ns) &&
                         mbar_wait_bounded(v_full, 0, a.wait_ns);
            if (ok) {
                tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < CH / 16; ++kk) {
                    const uint64_t ad = pd + (uint64_t)(((kk / 4) * M * 128 + (kk % 4) * 32) >> 4);
                    // V as B, MN-major: 64-dim slabs CH * 128 bytes apart (leading
                    // offset), 8-token atoms 1 KiB apart (stride offset)
                    const uint64_t bd = vd + (uint64_t)((kk * 16 * 128) >> 4);
                    umma_bf16(o_tmem, ad, bd, umma_idesc_bf16(M, D, true), kk > 0);
                }
                umma_commit(o_full);
                o_issued = true;
            }
            if (!ok) {
                raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
                failed = 1;
            }
            // nothing this thread issued may still run when TMEM is freed
            if (o_issued) (void)mbar_wait_bounded(o_full, 0, a.wait_ns);
            else if (s_issued)   // the last group committed covers every earlier MMA
                for (int g = NG - 1; g >= 0; --g)
                    if (mbar_wait_bounded(&s_full[g], 0, a.wait_ns)) break;
        }
    } else {
        // -------------------------------- softmax and epilogue: warps 0-3 --
        const int r = 32 * warp + lane;                   // this thread's query row / TMEM lane
        const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
        auto soft_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(32 * C::SOFT_WARPS) : "memory"); };
        // every softmax warp must agree before it depends on the others
        // (each agreement point has its own flags: a fast warp must not
        // overwrite flags a slow one is still reading)
        auto all_ok = [&](int point, bool mine) {
            int* f = okw + point * C::SOFT_WARPS;
            if (lane == 0) f[warp] = mine ? 1 : 0;
            soft_sync();
            int ok = 1;
#pragma unroll
            for (int w = 0; w < C::SOFT_WARPS; ++w) ok &= f[w];
            return ok != 0;
        };
        float m = -INFINITY, l = 0.f;
        // pass 1: the row's maximum over the chunk's prefix tokens (log2 units),
        // one 64-token group at a time as its S MMAs complete
        bool ok = true;
#pragma unroll 1
        for (int c = 0; c < CH / 64 && ok; ++c) {
            ok = __all_sync(FULL_MASK, mbar_wait_bounded(&s_full[c], 0, a.wait_ns));
            if (ok) {
                tc_fence_after_sync();
                float v0[32], v1[32];
                tmem_ld32(s_tmem + lane_off + 64 * c, v0);
                tmem_ld32(s_tmem + lane_off + 64 * c + 32, v1);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (64 * c + j < valid) m = fmaxf(m, v0[j] * a.scale_log2);
                    if (64 * c + 32 + j < valid) m = fmaxf(m, v1[j] * a.scale_log2);
                }
            }
        }
        if (ok) {
            // pass 2: p = 2^(x - m) into the P tile (bf16, 128-byte swizzle), sum of p;
            // 64 tokens = one slab row of 128 bytes per round trip
            const uint32_t prow = smem_addr(ks) + (uint32_t)r * 128;
#pragma unroll 1
            for (int c = 0; c < CH / 64; ++c) {
                float v[64];
                tmem_ld32(s_tmem + lane_off + 64 * c, *reinterpret_cast<float(*)[32]>(v));
                tmem_ld32(s_tmem + lane_off + 64 * c + 32,
                          *reinterpret_cast<float(*)[32]>(v + 32));
                tmem_ld_wait();
                uint32_t w[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int t = 64 * c + 2 * j;
                    const float p0 = t < valid ? exp2_approx(v[2 * j] * a.scale_log2 - m) : 0.f;
                    const float p1 =
                        t + 1 < valid ? exp2_approx(v[2 * j + 1] * a.scale_log2 - m) : 0.f;
                    l += p0 + p1;
                    w[j] = pack_bf16x2(p0, p1);
                }
                const uint32_t base = prow + (uint32_t)c * (M * 128);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t addr = base + (uint32_t)((q ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(w[4 * q]), "r"(w[4 * q + 1]), "r"(w[4 * q + 2]),
                                 "r"(w[4 * q + 3])
                                 : "memory");
                }
            }
            fence_proxy_async_smem();                   // P is read by the tensor cores
            tc_fence_before_sync();
            mbar_arrive(p_full);
            ok = __all_sync(FULL_MASK, mbar_wait_bounded(o_full, 0, a.wait_ns));
        }
        ok = all_ok(0, ok);
        if (!ok) {
            if (r == 0) {
                raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
                failed = 1;
            }
        } else {
            tc_fence_after_sync();
            // the row's output, OCOLS columns at a time: this thread stages
            // its row (padded rows, over the tiles no MMA or load uses any
            // more) and sends it to the workspace with one bulk copy
            float* os = reinterpret_cast<float*>(smem) + r * C::OSTRIDE;
            const int row = row0 + r;
            const bool mine = row < rows;
            const int seq = gs + row / G, h = kvh * G + row % G;
            const size_t slot = ((size_t)seq * a.num_heads + h) * a.slot_stride +
                                a.prefix_slot0 + chunk;
#pragma unroll 1
            for (int cb = 0; cb < D / C::OCOLS; ++cb) {
                if (cb > 0) bulk_wait_read();           // the staging row is free again
#pragma unroll
                for (int c = 0; c < C::OCOLS / 32; ++c) {
                    float t[32];
                    tmem_ld32(o_tmem + lane_off + cb * C::OCOLS + 32 * c, t);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<float4*>(os + 32 * c + 4 * j) =
                            make_float4(t[4 * j], t[4 * j + 1], t[4 * j + 2], t[4 * j + 3]);
                }
                if (mine) {
                    fence_proxy_async_smem();           // the bulk copy reads the row
                    bulk_store(a.ws_o + slot * D + cb * C::OCOLS, os, C::OCOLS * 4);
                    bulk_commit();
                }
            }
            if (mine) {
                a.ws_m[slot] = m;
                a.ws_l[slot] = l;
                bulk_wait();                            // complete before the CTA leaves
            }
        }
    }

    // ---------------- teardown: every role is done with TMEM and shared memory --
    tc_fence_before_sync();
    __syncthreads();
    if (failed && warp == C::PRODUCER && lane == 0) {
        // loads may still be in flight after a role gave up: wait (bounded) for them
        (void)mbar_wait_bounded(q_full, 0, a.wait_ns);
        for (int g = 0; g < NG; ++g) (void)mbar_wait_bounded(&k_full[g], 0, a.wait_ns);
        if (v_issued) (void)mbar_wait_bounded(v_full, 0, a.wait_ns);
    }
    if (warp == C::MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (failed) __syncthreads();                          // keep shared memory until the drain
}

}  // namespace pa
