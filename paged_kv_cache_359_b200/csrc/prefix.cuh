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
// CTA = (prefix chunk of CH = 256 tokens, kv head, group x 128-row block);
// S (CH columns) and O (head_dim columns) share the SM's 512 TMEM columns, so
// at head_dim 256 a CTA holds all of them.  Roles:
//  * producer warp: TMA loads of the CTA's 128 query rows (a 3-D box over
//    q [S][Hq][D]: members x G heads, row = member * G + head) and of the
//    chunk's K tiles in 64-token groups, all at once, one slot per group;
//    each group's V tiles go into its slot once the MMAs that read its K
//    are done; all 128-byte swizzled; a unit past the prefix is loaded from
//    outside the pool map, which TMA fills with zeros;
//  * MMA warp (one elected thread): S = Q K^T into TMEM (M = 128 rows,
//    N = 64 tokens per group as its K tiles land, K = head_dim), a commit
//    per group; then, group by group as its P and V tiles land, O += P V
//    into TMEM (M = 128, N = head_dim, K = 64 tokens, V read MN-major), a
//    commit per group that frees the group's P slot;
//  * four softmax warps, one TMEM lane (query row) per thread: the exact
//    maximum of the row's scores over the chunk (masked past the prefix),
//    then per group p = 2^(s * scale * log2 e - max), rounded to bf16, into
//    a ring of two swizzled P slots in Q's space, and the fp32 sum of p;
//    after the last MMA each thread stages its row's output in the freed
//    tiles and sends it with TMA bulk copies to the workspace slot
//    prefix_slot0 + chunk, with the row's maximum and sum; pa_decode's CTAs
//    for each sequence's own tokens merge these into the output.
// The CTA holds Q (or the P ring) and one chunk of K/V: 97 KB of shared
// memory at head_dim 128 (193 KB at 256, which leaves no room beside it).
// At head_dim 128, beside it on an SM the own-token pass fits three two-warp
// CTAs, or one four-warp CTA: an SM's registers sit in four per-quarter
// files, and this CTA's six warps take two of them twice.  Bounding the
// registers here so that two four-warp CTAs fit made the step no faster (the
// two passes then contend for the same SMs); a two-slot K/V ring (67 KB)
// waited on four rounds of loads.
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
    static constexpr int CH = 256;                     // chunk tokens
    static constexpr int U = CH / R;                   // units per chunk
    static constexpr int NG = CH / 64;                 // 64-token groups
    static constexpr int KSL = D / 64;                 // 64-dim slabs of a 128-byte-swizzled tile
    static constexpr int M = 128;                      // query rows per CTA
    static constexpr int Q_BYTES = KSL * M * 128;
    static constexpr int GROUP_BYTES = KSL * 64 * 128; // one 64-token group of K or V
    static constexpr int P_BYTES = M * 128;            // one 64-token group of P
    // region A: Q, then a ring of two P groups; region B: a slot per 64-token
    // group, which holds the group's K and then its V
    static constexpr int A_BYTES = Q_BYTES > 2 * P_BYTES ? Q_BYTES : 2 * P_BYTES;
    static constexpr int B_BYTES = NG * GROUP_BYTES;
    static constexpr int A_OFF = 0, B_OFF = A_BYTES;
    static constexpr int BAR_OFF = A_BYTES + B_BYTES;
    // q_full; k_full[NG], v_full[NG] (per group); p_full[2], pv_done[2] (per
    // P slot); s_full[NG] (S of group g done); o_full; then the TMEM address
    static constexpr int NBARS = 6 + 3 * NG;
    static constexpr int P_FULL = 1 + 2 * NG;         // index of p_full[0]
    static constexpr int SOFT_WARPS = 4;
    static constexpr int PRODUCER = SOFT_WARPS, MMA_WARP = SOFT_WARPS + 1;
    static constexpr int THREADS = (SOFT_WARPS + 2) * 32;
    // the output is staged OCOLS columns at a time, rows padded by 4 floats,
    // over the freed tiles
    static constexpr int OCOLS_MAX = D < 128 ? D : 128;
    static constexpr int OCOLS = M * (OCOLS_MAX + 4) * 4 <= BAR_OFF ? OCOLS_MAX : 64;
    static constexpr int OSTRIDE = OCOLS + 4;
    // barriers, the TMEM address, agreement flags, then alignment slack
    static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 16 + 2 * 4 * 4 + 1024;
    static constexpr int TMEM_COLS = 512;             // S at column 0, O at column CH
    static_assert(M * OSTRIDE * 4 <= BAR_OFF, "staged output fits the freed tiles");
    static_assert((BS % R == 0 || BS == 8) && D % 64 == 0, "shared-prefix shape");
    static_assert(CH + D <= TMEM_COLS, "S and O must fit TMEM");
    static_assert(NG >= 2, "a two-slot P ring");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

constexpr int PREFIX_ROWS_PER_CTA = 128;

// Tokens per prefix chunk (one CTA's share of the shared prefix).  At
// head_dim 256, 128-token chunks (two CTAs' worth of the SM's TMEM columns in
// one wave each) measured 0.0551 against 0.0657 ms per cascade step: twice
// the CTAs in two waves, and twice the partials to merge.
__host__ __device__ constexpr int prefix_chunk_tokens(int head_dim) {
    (void)head_dim;
    return 256;
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
    unsigned char* ra = smem + C::A_OFF;                  // Q, then the P ring
    unsigned char* rb = smem + C::B_OFF;                  // per group: K, then V
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;                          // [NG] per group slot
    uint64_t* v_full = k_full + NG;                       // [NG]
    uint64_t* p_full = v_full + NG;                       // [2]: the softmax warps wrote P
    uint64_t* pv_done = p_full + 2;                       // [2]: O += P V of the P slot's group done
    uint64_t* s_full = pv_done + 2;                       // [NG]: S of 64-token group g done
    uint64_t* o_full = s_full + NG;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
    int* okw = reinterpret_cast<int*>(tmem_slot + 4);             // [2][SOFT_WARPS]
    // set by a role that gave up, read by the others after the final barrier
    __shared__ int failed;

    if (threadIdx.x == 0) {
        failed = 0;
        for (int i = 0; i < C::NBARS; ++i)
            mbar_init(&bars[i], (i == C::P_FULL || i == C::P_FULL + 1) ? 32 * C::SOFT_WARPS : 1);
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
    int k_issued = 0, v_issued = 0;                       // producer lane 0: groups loaded

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
                tma_load_3d(ra + b * M * 128, &tm_q, q_full, 64 * b, kvh * G, gs + row0 / G);
            // group g (units 4g .. 4g+3 of the chunk) into slot g: unit jj
            // lands at row 16 jj of every 64-dim slab of the slot
            auto load_group = [&](const CUtensorMap* map, uint64_t* bar, int g) {
                unsigned char* base = rb + g * C::GROUP_BYTES;
                mbar_arrive_expect_tx(bar, C::GROUP_BYTES + a.tx_extra);
                for (int jj = 0; jj < 4; ++jj) {
                    const int u = u_begin + 4 * g + jj;
                    int id = a.num_blocks, id1 = a.num_blocks, rr = 0;
                    if (u < u_end) {                // the prefix is whole 16-token units
                        id = checked(__ldg(table + (u * R) / BS));
                        if (C::BOX_ROWS < R) id1 = checked(__ldg(table + (u * R) / BS + 1));
                        else rr = (u * R) % BS;
                    }
#pragma unroll
                    for (int b = 0; b < KSL; ++b) {
                        unsigned char* dst = base + b * (64 * 128) + jj * R * 128;
                        tma_load_4d(dst, map, bar, 64 * b, kvh, rr, id);
                        if (C::BOX_ROWS < R)
                            tma_load_4d(dst + C::BOX_ROWS * 128, map, bar, 64 * b, kvh, 0, id1);
                    }
                }
            };
            bool ok = true;
            // every K group at once; then each V group into its K group's slot
            // once the S MMAs of that group are done
            for (int g = 0; g < NG; ++g) {
                load_group(&tm_k, &k_full[g], g);
                k_issued = g + 1;
            }
            for (int g = 0; g < NG && ok; ++g) {
                ok = mbar_wait_bounded(&s_full[g], 0, a.wait_ns);
                if (ok) {
                    load_group(&tm_v, &v_full[g], g);
                    v_issued = g + 1;
                }
            }
            if (!ok) {
                raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
                failed = 1;
            }
        }
    } else if (warp == C::MMA_WARP) {
        // --------------------------------------------- MMA issuer (lane 0) --
        if (lane == 0) {
            const uint32_t a0 = smem_addr(ra), b0 = smem_addr(rb);
            // base descriptors; a step's operand is the base plus a byte
            // offset (>> 4) added to the start-address field, which stays
            // inside its 14 bits for any shared-memory address
            const uint64_t qd = sw128_desc(a0, 16, 1024);
            uint64_t* last = nullptr;                     // the last commit issued
            uint32_t last_parity = 0;
            bool ok = mbar_wait_bounded(q_full, 0, a.wait_ns);
            // S = Q K^T, one 64-token group at a time as its K tiles land
            for (int g = 0; g < NG && ok; ++g) {
                ok = mbar_wait_bounded(&k_full[g], 0, a.wait_ns);
                if (!ok) break;
                tc_fence_after_sync();
                const uint64_t kd = sw128_desc(b0 + g * C::GROUP_BYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4 * KSL; ++kk) {
                    const uint64_t ad = qd + (uint64_t)(((kk / 4) * M * 128 + (kk % 4) * 32) >> 4);
                    const uint64_t bd = kd + (uint64_t)(((kk / 4) * 64 * 128 + (kk % 4) * 32) >> 4);
                    umma_bf16(s_tmem + 64 * g, ad, bd, umma_idesc_bf16(M, 64, false), kk > 0);
                }
                umma_commit(&s_full[g]);              // the softmax starts on this group
                last = &s_full[g];
                last_parity = 0;
            }
            // O = P V, group by group as P and V land (P K-major; V MN-major:
            // 64-dim slabs 64 * 128 bytes apart as the leading offset,
            // 8-token atoms 1 KiB apart as the stride offset)
            for (int g = 0; g < NG && ok; ++g) {
                ok = mbar_wait_bounded(&p_full[g % 2], (g / 2) & 1, a.wait_ns) &&
                     mbar_wait_bounded(&v_full[g], 0, a.wait_ns);
                if (!ok) break;
                tc_fence_after_sync();
                const uint64_t pd = sw128_desc(a0 + (g % 2) * C::P_BYTES, 16, 1024);
                const uint64_t vd = sw128_desc(b0 + g * C::GROUP_BYTES, 64 * 128, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = pd + (uint64_t)((kk * 32) >> 4);
                    const uint64_t bd = vd + (uint64_t)((kk * 16 * 128) >> 4);
                    umma_bf16(o_tmem, ad, bd, umma_idesc_bf16(M, D, true), g > 0 || kk > 0);
                }
                umma_commit(&pv_done[g % 2]);         // the P slot is free again
                last = &pv_done[g % 2];
                last_parity = (g / 2) & 1;
            }
            if (ok) {
                umma_commit(o_full);
                last = o_full;
                last_parity = 0;
            } else {
                raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
                failed = 1;
            }
            // nothing this thread issued may still run when TMEM is freed (the
            // last commit covers every earlier MMA)
            if (last) (void)mbar_wait_bounded(last, last_parity, a.wait_ns);
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
            // pass 2: p = 2^(x - m) into the P ring (bf16, 128-byte swizzle), sum
            // of p; a group of 64 tokens is one slab row of 128 bytes, written
            // once the slot's previous group has been multiplied
            const uint32_t prow = smem_addr(ra) + (uint32_t)r * 128;
#pragma unroll 1
            for (int c = 0; c < CH / 64 && ok; ++c) {
                if (c >= 2) {
                    ok = __all_sync(FULL_MASK, mbar_wait_bounded(&pv_done[c % 2],
                                                                 ((c - 2) / 2) & 1, a.wait_ns));
                    if (!ok) break;
                }
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
                const uint32_t base = prow + (uint32_t)(c % 2) * C::P_BYTES;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t addr = base + (uint32_t)((q ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(w[4 * q]), "r"(w[4 * q + 1]), "r"(w[4 * q + 2]),
                                 "r"(w[4 * q + 3])
                                 : "memory");
                }
                fence_proxy_async_smem();               // P is read by the tensor cores
                tc_fence_before_sync();
                mbar_arrive(&p_full[c % 2]);
            }
            if (ok) ok = __all_sync(FULL_MASK, mbar_wait_bounded(o_full, 0, a.wait_ns));
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
        // loads may still be in flight after a role gave up: wait (bounded) for
        // them (a V group is loaded only after its slot's K group landed)
        (void)mbar_wait_bounded(q_full, 0, a.wait_ns);
        for (int g = 0; g < k_issued; ++g) (void)mbar_wait_bounded(&k_full[g], 0, a.wait_ns);
        for (int g = 0; g < v_issued; ++g) (void)mbar_wait_bounded(&v_full[g], 0, a.wait_ns);
    }
    if (warp == C::MMA_WARP) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (failed) __syncthreads();                          // keep shared memory until the drain
}

}  // namespace pa
