// Paged decode attention kernels for sm_100a.
//
// What is computed ("vLLM内存管理与PagedAttention精讲" ch.2 §2.5; "VLLM中
// PagedAttention如何降低显存碎片？" §三 items 4-6, 9): for every sequence and
// query head, softmax(scale * q.K^T) V over the sequence's tokens, where token
// t sits in physical block table[t / block_size] at row t % block_size and
// query head h reads kv head h / G (G = num_heads / num_kv_heads).
//
// How (B200 design, not the pages' A100 sketch):
//  * One CTA per (sequence, kv head[, partition or cluster rank]); all G
//    query heads of the kv group share every K/V tile the CTA loads.
//  * Work unit = R consecutive tokens of one block for one kv head: a K tile
//    and a V tile of R rows x head_dim, each one 4-D TMA box
//    {head_dim, 1, R, 1} over the cache viewed as
//    [num_blocks][block_size][kv_heads][head_dim].  R is chosen so a tile is
//    at most 4 KiB; with block_size 16 / head_dim 128 / bf16 a unit is one
//    whole block.
//  * Each of the NW warps owns a private ring of DEPTH stages with its own
//    mbarriers: lane 0 issues the TMA loads DEPTH units ahead, all lanes wait
//    on the stage's barrier (bounded), compute, and lane 0 refills the stage.
//    Warps take units round-robin, so every warp streams independently and
//    there is no CTA-wide barrier in the main loop.
//  * Block-table lookups are hoisted: every 32 units a warp loads the next 32
//    block ids with one coalesced read (one id per lane) and hands them to
//    lane 0 with a shuffle.
//  * QK: a K row is spread over LPR lanes, 16 bytes per lane; each lane forms
//    partial dot products for all G heads of its rows, then a butterfly
//    reduce-scatter across the LPR lanes leaves every lane holding complete
//    scores for a few (row, head) pairs.
//  * Online softmax in fp32, in log2 units (q is pre-scaled by
//    scale * log2 e), with a lazy running max: the accumulator is only
//    rescaled when a score exceeds the current max by more than 2^8, which
//    keeps exp2 arguments bounded and the result exact up to rounding.
//  * PV: probabilities go through a tiny per-warp shared buffer so each lane
//    reads the weights of its own rows, then fp32 FMAs into registers.
//  * Warps merge through shared memory; the CTAs of a cluster (pa_decode on
//    long sequences) merge through distributed shared memory; split-K
//    partitions write (max, sum, unnormalised output) to a workspace for the
//    log-sum-exp reduce kernel.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace pa {

namespace cg = cooperative_groups;

constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units: rescale when a score tops the max by 2^8

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

struct DecodeArgs {
    void* out;                    // [S, Hq, D]
    const void* q;                // [S, Hq, D]
    const int32_t* block_tables;  // [S, max_blocks]
    const int32_t* context_lens;  // [S]
    float* ws_m;                  // split: [S, Hq, max_parts] running max (log2 units)
    float* ws_l;                  // split: [S, Hq, max_parts] sum of exponentials
    float* ws_o;                  // split: [S, Hq, max_parts, D] unnormalised output
    unsigned* err;                // device error word
    float scale_log2;             // scale * log2(e)
    int max_blocks;
    int max_tokens;               // max_blocks * block_size
    int num_heads;
    int num_kv_heads;
    int num_blocks;
    int part_tokens;              // split: partition size in tokens
    int max_parts;                // split: partitions per (sequence, head) in the workspace
};

enum class Mode { Decode, Split };

template <typename T, int D, int BS, int G>
struct Geom {
    static constexpr int ES = (int)sizeof(T);
    static constexpr int VEC = 16 / ES;                 // elements per 16-byte vector
    static constexpr int VPR = D / VEC;                 // vectors per K/V row
    static constexpr int LPR = cmin(VPR, 32);           // lanes per row
    static constexpr int VPL = VPR / LPR;               // vectors per lane per row
    static constexpr int RPP = 32 / LPR;                // rows per warp pass
    static constexpr int R = cmin(BS, cmax(RPP, 4096 / (D * ES)));   // rows per unit
    static constexpr int PASSES = R / RPP;
    static constexpr int N = PASSES * G;                // partial scores per lane per unit
    static constexpr int LOG_LPR = ilog2(LPR);
    static constexpr int RS = cmin(LOG_LPR, ilog2(N));  // reduce-scatter steps
    static constexpr int NH = N >> RS;                  // scores held per lane afterwards
    static constexpr int DUP = LPR >> RS;               // lanes holding the same score
    static constexpr int UNIT_BYTES = R * D * ES;       // one K (or V) tile
    static constexpr int STAGE_BYTES = 2 * UNIT_BYTES;
    static constexpr int NW = 4;                        // warps per CTA
    static constexpr int DEPTH = cmin(8, cmax(3, 24576 / STAGE_BYTES));
    static constexpr int STAGE_REGION = NW * DEPTH * STAGE_BYTES;
    static constexpr int MERGE_FLOATS = (NW + 1) * G * (D + 2);
    static constexpr int MAIN_REGION = cmax(STAGE_REGION, MERGE_FLOATS * 4);
    static constexpr int PBUF_BYTES = NW * R * G * 4;
    static constexpr int BAR_OFFSET = MAIN_REGION + PBUF_BYTES;
    static constexpr int SMEM_BYTES = BAR_OFFSET + NW * DEPTH * 8;

    static_assert(D % VEC == 0 && VPR % LPR == 0, "head_dim must be a multiple of 16 bytes");
    static_assert(BS % R == 0 && R % RPP == 0, "unit rows must tile the block");
    static_assert((N & (N - 1)) == 0, "power-of-two score count");
    static_assert(MAIN_REGION % 16 == 0 && PBUF_BYTES % 16 == 0, "alignment");
};

// Process one unit (R rows of K and V) for one warp.
template <typename T, int D, int BS, int G, bool MASKED>
__device__ __forceinline__ void process_unit(
    const T* __restrict__ ks, const T* __restrict__ vs, float* __restrict__ pbuf, int valid,
    int lane, const float (&qf)[G][Geom<T, D, BS, G>::VPL][Geom<T, D, BS, G>::VEC],
    float (&acc)[G][Geom<T, D, BS, G>::VPL][Geom<T, D, BS, G>::VEC], float (&m)[G],
    float (&mh)[Geom<T, D, BS, G>::NH], float (&lh)[Geom<T, D, BS, G>::NH],
    const int (&hg)[Geom<T, D, BS, G>::NH], const int (&hrow)[Geom<T, D, BS, G>::NH]) {
    using Gm = Geom<T, D, BS, G>;
    constexpr int VEC = Gm::VEC, VPL = Gm::VPL, LPR = Gm::LPR, RPP = Gm::RPP;
    constexpr int PASSES = Gm::PASSES, N = Gm::N, NH = Gm::NH;
    const int c = lane % LPR;
    const int r = lane / LPR;

    // ---- partial dot products q_g . k_row over this lane's slice of D ----
    float x[N];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int row = p * RPP + r;
        float kf[VPL][VEC];
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            const uint4 u = *reinterpret_cast<const uint4*>(ks + row * D + (v * LPR + c) * VEC);
            Vec16<T>::to_float(u, kf[v]);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float s = 0.f;
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < VEC; ++e) s = fmaf(qf[g][v][e], kf[v][e], s);
            x[p * G + g] = s;
        }
    }

    // ---- butterfly reduce-scatter across the LPR lanes of a row ----
#pragma unroll
    for (int k = 0; k < Gm::RS; ++k) {
        const int half = N >> (k + 1);
        const bool upper = (lane >> k) & 1;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float lo = x[i], hi = x[i + half];
            const float send = upper ? lo : hi;
            const float keep = upper ? hi : lo;
            x[i] = keep + __shfl_xor_sync(FULL_MASK, send, 1 << k);
        }
    }
#pragma unroll
    for (int k = Gm::RS; k < Gm::LOG_LPR; ++k) x[0] += __shfl_xor_sync(FULL_MASK, x[0], 1 << k);

    float sc[NH];
#pragma unroll
    for (int j = 0; j < NH; ++j) {
        sc[j] = x[j];
        if (MASKED && hrow[j] >= valid) sc[j] = -INFINITY;
    }

    // ---- lazy running max ----
    bool grow = false;
#pragma unroll
    for (int j = 0; j < NH; ++j) grow |= sc[j] > mh[j] + RESCALE_THRESHOLD;
    if (__any_sync(FULL_MASK, grow)) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float lm = -INFINITY;
#pragma unroll
            for (int j = 0; j < NH; ++j)
                if (hg[j] == g) lm = fmaxf(lm, sc[j]);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
                lm = fmaxf(lm, __shfl_xor_sync(FULL_MASK, lm, off));
            const float mn = fmaxf(m[g], lm);
            const float alpha = exp2_approx(m[g] - mn);
            m[g] = mn;
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[g][v][e] *= alpha;
#pragma unroll
            for (int j = 0; j < NH; ++j)
                if (hg[j] == g) {
                    lh[j] *= alpha;
                    mh[j] = mn;
                }
        }
    }

    // ---- probabilities: keep the running sum, publish to the warp ----
#pragma unroll
    for (int j = 0; j < NH; ++j) {
        const float pj = exp2_approx(sc[j] - mh[j]);
        lh[j] += pj;
        pbuf[hrow[j] * G + hg[j]] = pj;
    }
    __syncwarp();

    // ---- PV ----
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int row = p * RPP + r;
        float pv[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
            for (int g = 0; g < G; g += 4) {
                const float4 w = *reinterpret_cast<const float4*>(pbuf + row * G + g);
                pv[g] = w.x; pv[g + 1] = w.y; pv[g + 2] = w.z; pv[g + 3] = w.w;
            }
        } else if constexpr (G == 2) {
            const float2 w = *reinterpret_cast<const float2*>(pbuf + row * G);
            pv[0] = w.x; pv[1] = w.y;
        } else {
            pv[0] = pbuf[row];
        }
        float vf[VPL][VEC];
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            const uint4 u = *reinterpret_cast<const uint4*>(vs + row * D + (v * LPR + c) * VEC);
            Vec16<T>::to_float(u, vf[v]);
        }
        if (MASKED && row >= valid) {
            // rows past the end of the sequence may hold anything (NaN poison)
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < VEC; ++e) vf[v][e] = 0.f;
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[g][v][e] = fmaf(pv[g], vf[v][e], acc[g][v][e]);
    }
    __syncwarp();
}

template <typename T, int D, int BS, int G, Mode MODE>
__global__ void __launch_bounds__(Geom<T, D, BS, G>::NW * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
    using Gm = Geom<T, D, BS, G>;
    constexpr int NW = Gm::NW, DEPTH = Gm::DEPTH, R = Gm::R, VEC = Gm::VEC, VPL = Gm::VPL;
    constexpr int LPR = Gm::LPR, NH = Gm::NH, N = Gm::N;
    constexpr int NT = NW * 32;

    const int seq = blockIdx.z;
    const int kvh = blockIdx.y;
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    // ---- this CTA's share of the sequence, in units of R tokens ----
    int L = a.context_lens[seq];
    const int cap = a.max_tokens;
    if (L < 0 || L > cap) {
        if (threadIdx.x == 0) raise_error(a.err, PA_DEVERR_CONTEXT_LEN);
        L = L < 0 ? 0 : cap;
    }
    const int total_units = (L + R - 1) / R;
    int u_begin = 0, u_end = total_units, ctas = 1, crank = 0, part = 0, nparts = 1;
    if constexpr (MODE == Mode::Split) {
        part = blockIdx.x;
        nparts = (L + a.part_tokens - 1) / a.part_tokens;
        if (part >= cmax(nparts, 1)) return;            // whole CTA, before any barrier
        if (nparts > a.max_parts) {
            if (threadIdx.x == 0 && part == 0) raise_error(a.err, PA_DEVERR_WORKSPACE);
            if (part > 0) return;
            nparts = 1;                                  // degrade: partition 0 covers the rest
            u_begin = 0;
        } else {
            u_begin = part * (a.part_tokens / R);
            u_end = cmin(u_begin + a.part_tokens / R, total_units);
        }
    } else {
        ctas = gridDim.x;
        crank = blockIdx.x;
    }
    const int ustride = ctas * NW;
    const int first = u_begin + crank + ctas * warp;
    const int nk = first < u_end ? (u_end - first + ustride - 1) / ustride : 0;

    extern __shared__ __align__(128) unsigned char smem[];
    T* stage_base = reinterpret_cast<T*>(smem) + (size_t)warp * DEPTH * (2 * R * D);
    float* pbuf = reinterpret_cast<float*>(smem + Gm::MAIN_REGION) + warp * R * G;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Gm::BAR_OFFSET) + warp * DEPTH;

    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < DEPTH; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        if (warp == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
        }
    }
    __syncwarp();

    const int c = lane % LPR;
    const int r = lane / LPR;

    // ---- queries of the kv group, pre-scaled into log2 units ----
    float qf[G][VPL][VEC];
    {
        const T* qb = reinterpret_cast<const T*>(a.q) +
                      ((size_t)seq * a.num_heads + (size_t)kvh * G) * D;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const uint4 u = *reinterpret_cast<const uint4*>(qb + g * D + (v * LPR + c) * VEC);
                Vec16<T>::to_float(u, qf[g][v]);
#pragma unroll
                for (int e = 0; e < VEC; ++e) qf[g][v][e] *= a.scale_log2;
            }
    }

    // ---- hoisted block-table window: lane i holds the block of unit k0+i ----
    const int32_t* table = a.block_tables + (size_t)seq * a.max_blocks;
    int win = 0;
    auto load_window = [&](int k0) {
        const int k = k0 + lane;
        int id = 0;
        if (k < nk) {
            const int u = first + ustride * k;
            id = __ldg(table + (u * R) / BS);
            if (id < 0 || id >= a.num_blocks) {
                raise_error(a.err, PA_DEVERR_BLOCK_ID);
                id = a.num_blocks;        // out of the tensor map: TMA fills zeros
            }
        }
        win = id;
    };
    auto issue = [&](int k, int id) {    // lane 0 only
        const int s = k % DEPTH;
        T* kdst = stage_base + (size_t)s * (2 * R * D);
        const int u = first + ustride * k;
        const int row0 = (u * R) % BS;
        mbar_arrive_expect_tx(&bars[s], Gm::STAGE_BYTES);
        tma_load_4d(kdst, &tm_k, &bars[s], 0, kvh, row0, id);
        tma_load_4d(kdst + R * D, &tm_v, &bars[s], 0, kvh, row0, id);
    };

    load_window(0);
    const int pro = cmin(DEPTH, nk);
    for (int k = 0; k < pro; ++k) {
        const int id = __shfl_sync(FULL_MASK, win, k);
        if (lane == 0) issue(k, id);
    }

    // ---- per-lane softmax state ----
    float m[G], acc[G][VPL][VEC], mh[NH], lh[NH];
    int hg[NH], hrow[NH];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
#pragma unroll
        for (int v = 0; v < VPL; ++v)
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[g][v][e] = 0.f;
    }
    {
        int off = 0;
#pragma unroll
        for (int k = 0; k < Gm::RS; ++k) off += ((lane >> k) & 1) * (N >> (k + 1));
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            const int gi = j + off;
            hg[j] = gi % G;
            hrow[j] = (gi / G) * Gm::RPP + r;
            mh[j] = -INFINITY;
            lh[j] = 0.f;
        }
    }

    // ---- main loop over this warp's units ----
    int k = 0;
    bool failed = false;
    for (; k < nk; ++k) {
        const int s = k % DEPTH;
        const uint32_t parity = (k / DEPTH) & 1;
        const bool landed = __all_sync(FULL_MASK, mbar_wait_bounded(&bars[s], parity));
        if (!landed) {
            failed = true;
            break;
        }
        const T* ks = stage_base + (size_t)s * (2 * R * D);
        const int u = first + ustride * k;
        const int valid = cmin(R, L - u * R);
        if (valid == R)
            process_unit<T, D, BS, G, false>(ks, ks + R * D, pbuf, valid, lane, qf, acc, m, mh,
                                             lh, hg, hrow);
        else
            process_unit<T, D, BS, G, true>(ks, ks + R * D, pbuf, valid, lane, qf, acc, m, mh,
                                            lh, hg, hrow);
        const int kn = k + DEPTH;
        if (kn < nk) {
            if (kn % 32 == 0) load_window(kn);
            const int id = __shfl_sync(FULL_MASK, win, kn % 32);
            if (lane == 0) issue(kn, id);
        }
    }
    if (failed) {
        // A load never landed: record it, wait (bounded) for this warp's
        // other loads in flight so none lands after the CTA is gone, and
        // contribute nothing.
        if (lane == 0) raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
        const int issued = cmin(nk, k + DEPTH);
        for (int kk = k + 1; kk < issued; ++kk)
            (void)mbar_wait_bounded(&bars[kk % DEPTH], (kk / DEPTH) & 1);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[g][v][e] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < NH; ++j) lh[j] = 0.f;
    }

    // ---- finish the warp: sum rows across row groups, sums per head ----
#pragma unroll
    for (int kk = Gm::LOG_LPR; kk < 5; ++kk)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                    acc[g][v][e] += __shfl_xor_sync(FULL_MASK, acc[g][v][e], 1 << kk);
    float lsum[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float t = 0.f;
#pragma unroll
        for (int j = 0; j < NH; ++j)
            if (hg[j] == g) t += lh[j];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) t += __shfl_xor_sync(FULL_MASK, t, off);
        lsum[g] = t * (1.0f / Gm::DUP);
    }

    // ---- merge the warps (the merge area overlays the stage ring) ----
    __syncthreads();
    float* wm = reinterpret_cast<float*>(smem);     // [NW][G]
    float* wl = wm + NW * G;                         // [NW][G]
    float* wacc = wl + NW * G;                       // [NW][G][D]
    float* xch = wacc + NW * G * D;                  // [G] max, [G] sum, [G][D] acc
    if (lane == 0)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            wm[warp * G + g] = m[g];
            wl[warp * G + g] = lsum[g];
        }
    if (r == 0)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                    wacc[(warp * G + g) * D + (v * LPR + c) * VEC + e] = acc[g][v][e];
    __syncthreads();

    T* out = reinterpret_cast<T*>(a.out);
    const size_t head0 = (size_t)seq * a.num_heads + (size_t)kvh * G;
    const bool cluster_merge = MODE == Mode::Decode && ctas > 1;
    for (int idx = threadIdx.x; idx < G * D; idx += NT) {
        const int g = idx / D, d = idx % D;
        float big = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) big = fmaxf(big, wm[w * G + g]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float mw = wm[w * G + g];
            const float e = mw == -INFINITY ? 0.f : exp2_approx(mw - big);
            num = fmaf(e, wacc[(w * G + g) * D + d], num);
            den = fmaf(e, wl[w * G + g], den);
        }
        if (cluster_merge) {
            if (d == 0) {
                xch[g] = big;
                xch[G + g] = den;
            }
            xch[2 * G + g * D + d] = num;
        } else if (MODE == Mode::Split && nparts > 1) {
            const size_t slot = (head0 + g) * a.max_parts + part;
            if (d == 0) {
                a.ws_m[slot] = big;
                a.ws_l[slot] = den;
            }
            a.ws_o[slot * D + d] = num;
        } else {
            store_out(out + (head0 + g) * D + d, den > 0.f ? num / den : 0.f);
        }
    }

    if constexpr (MODE == Mode::Decode) {
        if (cluster_merge) {
            cg::cluster_group cluster = cg::this_cluster();
            cluster.sync();                              // every rank's xch is written
            if (cluster.block_rank() == 0) {
                for (int idx = threadIdx.x; idx < G * D; idx += NT) {
                    const int g = idx / D, d = idx % D;
                    float big = -INFINITY;
                    for (int rk = 0; rk < ctas; ++rk)
                        big = fmaxf(big, cluster.map_shared_rank(xch, rk)[g]);
                    float num = 0.f, den = 0.f;
                    for (int rk = 0; rk < ctas; ++rk) {
                        const float* rx = cluster.map_shared_rank(xch, rk);
                        const float mr = rx[g];
                        const float e = mr == -INFINITY ? 0.f : exp2_approx(mr - big);
                        num = fmaf(e, rx[2 * G + g * D + d], num);
                        den = fmaf(e, rx[G + g], den);
                    }
                    store_out(out + (head0 + g) * D + d, den > 0.f ? num / den : 0.f);
                }
            }
            cluster.sync();                              // keep xch alive until rank 0 is done
        }
    }
}

// ---- log-sum-exp merge of split partitions ----
// grid (num_seqs * num_heads, D / 32), 256 threads: warp w folds partitions
// w, w+8, ...; lane = one of 32 dimensions.
template <typename T, int D>
__global__ void __launch_bounds__(256) lse_reduce_kernel(const DecodeArgs a) {
    const int sh = blockIdx.x;
    const int seq = sh / a.num_heads;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    int L = a.context_lens[seq];
    L = L < 0 ? 0 : cmin(L, a.max_tokens);
    const int nparts = (L + a.part_tokens - 1) / a.part_tokens;
    if (nparts <= 1 || nparts > a.max_parts) return;   // written directly by the partition kernel
    const float* m = a.ws_m + (size_t)sh * a.max_parts;
    const float* l = a.ws_l + (size_t)sh * a.max_parts;
    const float* o = a.ws_o + (size_t)sh * a.max_parts * D;

    __shared__ float red[8];
    __shared__ float part_num[8][32];
    float big = -INFINITY;
    for (int p = threadIdx.x; p < nparts; p += 256) big = fmaxf(big, m[p]);
    for (int off = 16; off >= 1; off >>= 1) big = fmaxf(big, __shfl_xor_sync(FULL_MASK, big, off));
    if (lane == 0) red[warp] = big;
    __syncthreads();
    big = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) big = fmaxf(big, red[w]);
    __syncthreads();
    float den = 0.f;
    for (int p = threadIdx.x; p < nparts; p += 256) den += exp2_approx(m[p] - big) * l[p];
    for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(FULL_MASK, den, off);
    if (lane == 0) red[warp] = den;
    __syncthreads();
    den = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) den += red[w];

    const int d = blockIdx.y * 32 + lane;
    float num = 0.f;
    for (int p = warp; p < nparts; p += 8) num = fmaf(exp2_approx(m[p] - big), o[(size_t)p * D + d], num);
    part_num[warp][lane] = num;
    __syncthreads();
    if (warp == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += part_num[w][lane];
        store_out(reinterpret_cast<T*>(a.out) + (size_t)sh * D + d, den > 0.f ? t / den : 0.f);
    }
}

}  // namespace pa
