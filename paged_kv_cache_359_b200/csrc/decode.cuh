// Paged decode attention kernels for sm_100a.
//
// What is computed ("vLLM内存管理与PagedAttention精讲" ch.2 §2.5; "VLLM中
// PagedAttention如何降低显存碎片？" §三 items 4-6, 9): for every sequence and
// query head, softmax(scale * q.K^T) V over the sequence's tokens, where token
// t sits in physical block table[t / block_size] at row t % block_size and
// query head h reads kv head h / G (G = num_heads / num_kv_heads).
//
// How (B200 design, not the pages' A100 sketch):
//  * Work item = (sequence, kv head): all G query heads of the kv group share
//    every K/V tile the CTA loads.  pa_decode launches one CTA per item and
//    CTA b finds, by a warp search over the context lengths, the item at
//    position b of the longest-first list, so the hardware block scheduler
//    starts the long sequences first and back-fills SMs with short ones.
//    With few items a cluster of CTAs shares one item instead and merges
//    through distributed shared memory; pa_decode_split gives every fixed
//    token partition its own CTA and merges partitions with a log-sum-exp
//    reduce kernel.
//  * Unit = R consecutive tokens of one block for one kv head: a K tile and
//    a V tile, each loaded by 4-D TMA boxes over the cache viewed as
//    [num_blocks][block_size][kv_heads][head_dim].
//  * Each of the NW warps owns a private ring of DEPTH stages with its own
//    mbarriers: lane 0 issues the TMA loads DEPTH units ahead, all lanes wait
//    (bounded), compute, and lane 0 refills the stage.  Warps take units
//    round-robin and stream independently; no CTA-wide barrier in the loop.
//  * Block-table lookups are hoisted: every 32 units a warp loads the next 32
//    block ids with one coalesced read and hands them to lane 0 by shuffle.
//  * Online softmax in fp32, in log2 units, with a lazy running max: the
//    accumulators are only rescaled when a score tops the current max by
//    more than 2^8, which bounds every exp2 argument and keeps the result
//    exact up to rounding.
//  * Two unit policies.  MmaUnit (bf16, R = 16): QK^T and PV on the
//    tensor cores with mma.sync m16n8k16 -- the G query rows of the group
//    form the M side (padded to 16), tokens and head_dim the N/K sides; tiles
//    arrive 128B-swizzled so ldmatrix reads them without bank conflicts.
//    CoreUnit (fp32 caches, block 8): fp32 FMAs with 16-byte loads and a
//    butterfly reduce-scatter across the lanes of a row.
#pragma once

#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"

namespace pa {

namespace cg = cooperative_groups;

constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units
constexpr int MAX_SORT = 1024;              // longest-first order up to this many sequences

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

// pa_decode schedules.  LPT: one CTA per (sequence, kv head), CTA b runs the
// item at position b of the longest-first list, so the hardware block
// scheduler hands out the longest items first and back-fills SMs greedily
// (longest-processing-time-first list scheduling).  CLUSTER: several CTAs
// per item, merged through distributed shared memory (few, long items).
enum Sched { SCHED_CLUSTER = 0, SCHED_LPT = 2 };

struct DecodeArgs {
    void* out;                    // [S, Hq, D]
    const void* q;                // [S, Hq, D]
    const int32_t* block_tables;  // [S, max_blocks]
    const int32_t* context_lens;  // [S]
    float* ws_m;                  // split: [S, Hq, max_parts] running max (log2 units)
    float* ws_l;                  // split: [S, Hq, max_parts] sum of exponentials
    float* ws_o;                  // split: [S, Hq, max_parts, D] unnormalised output
    // split reduce over reduce_chunks chunks of partitions per (sequence,
    // head): per chunk (sum of weighted outputs [D], sum of weights), then the
    // last chunk to arrive combines them (arrival counts zeroed by partition 0)
    float* ws_part;               // [S * Hq, reduce_chunks, D + 4]: sums [D], weight sum
    unsigned* ws_cnt;             // [S * Hq]
    int reduce_chunks;
    unsigned* err;                // device error word
    unsigned long long wait_ns;   // limit of every pipeline wait
    // test-only (PA_OPT_TEST_UNDERFED_STAGES): extra bytes armed on every
    // stage barrier beyond what its loads deliver, so its phase never
    // completes and each wait runs out; 0 in normal use
    unsigned tx_extra;
    float scale_log2;             // scale * log2(e)
    int num_seqs;
    int max_blocks;
    int max_tokens;               // max_blocks * block_size
    int num_heads;
    int num_kv_heads;
    int num_blocks;
    int part_tokens;              // split: partition size in tokens
    int max_parts;                // split: partitions per (sequence, head) in the workspace
    int sched;                    // pa_decode: SCHED_CLUSTER or SCHED_LPT
    // fused append (pa_decode_append): the new token of sequence s, rows
    // new_k/new_v [S, Hk, D], goes to slot new_slots[s] (-1: none) before
    // the sequence is read; null when not appending
    const void* new_k;
    const void* new_v;
    const int64_t* new_slots;
    void* k_cache;                // written only by the fused append
    void* v_cache;
    // pa_decode_step: the step's mapping update fused in.  Sequence s's last
    // block is the new slot's block (new_slots[s] / block_size), not its
    // table entry, and the CTA of kv head 0 writes it into the table
    // (block_tables, writable); null otherwise
    int32_t* table_out;
    // shared-prefix decode: sequences [group_starts[g], group_starts[g+1])
    // share their first group_prefix[g] tokens.  The shared pass leaves one
    // (max, sum, unnormalised output) per (sequence, head, prefix chunk) at
    // workspace slots [prefix_slot0, prefix_slot0 + ceil(prefix / chunk_tokens));
    // pa_decode's CTAs then cover only each sequence's own tokens and merge
    // those chunks into their output.  null: off
    const int32_t* group_starts;
    const int32_t* group_prefix;
    int num_groups;
    int chunk_tokens;
    int prefix_slot0;
    int slot_stride;              // workspace slots per (sequence, head)
};

// Group of sequence `seq` (binary search over group_starts) and its shared
// prefix length; 0 when no groups are given.
__device__ __forceinline__ int shared_prefix_of(const DecodeArgs& a, int seq) {
    if (!a.group_starts) return 0;
    int lo = 0, hi = a.num_groups;           // group_starts[lo] <= seq < group_starts[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(a.group_starts + mid) <= seq) lo = mid; else hi = mid;
    }
    return __ldg(a.group_prefix + lo);
}

// Warp-wide selection: lane l holds values get(0..PL-1) of entries l, l+32,
// ... (-1 for no entry, else >= 0).  Returns the entry at rank r of the list
// sorted by (value descending, entry ascending), and its value in `value`:
// a binary search for the value v at rank r (counts by warp reduction), then
// the k-th entry equal to v in entry order by ballots.  r must be below the
// number of entries.
template <int PL, class Get>
__device__ __forceinline__ int rank_select(Get&& get, int r, int lane, int& value) {
    int top = 0;
#pragma unroll
    for (int j = 0; j < PL; ++j) top = max(top, get(j));
    top = (int)__reduce_max_sync(FULL_MASK, (unsigned)top);
    int lo = 0, hi = top + 1;            // count(v >= lo) > r >= count(v >= hi)
    while (hi - lo > 1) {
        const int mid = lo + (hi - lo) / 2;
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < PL; ++j) cnt += get(j) >= mid;
        if ((int)__reduce_add_sync(FULL_MASK, (unsigned)cnt) > r)
            lo = mid;
        else
            hi = mid;
    }
    int gt = 0;
#pragma unroll
    for (int j = 0; j < PL; ++j) gt += get(j) > lo;
    const int k = r - (int)__reduce_add_sync(FULL_MASK, (unsigned)gt);
    int base = 0, found = -1;
#pragma unroll
    for (int j = 0; j < PL; ++j) {
        const bool eq = get(j) == lo;
        const unsigned ball = __ballot_sync(FULL_MASK, eq);
        const int before = __popc(ball & ((1u << lane) - 1u));
        if (eq && base + before == k) found = lane + 32 * j;
        base += __popc(ball);
    }
    value = lo;
    return (int)__reduce_max_sync(FULL_MASK, (unsigned)(found + 1)) - 1;
}

// Fused append in two phases, so that the loads of both go out before
// anything waits on them: append_load reads the new token's slot and this
// thread's share (at most two 16-byte vectors: vectors j and j + NT of the
// key | value row pair of kv head kvh) of the new rows; append_store writes
// them at the slot and makes the writes visible to the CTA's own TMA loads.
// The caller follows with a CTA barrier.  Only this sequence reads the new
// token's block (a shared block is copied before it is written), so no
// other CTA can race with the write.
struct AppendLoad {
    int64_t slot;
    uint4 x[2];
};

template <typename T, int D, int NT>
__device__ __forceinline__ AppendLoad append_load(const DecodeArgs& a, int seq, int kvh) {
    constexpr int NV = D * (int)sizeof(T) / 16;        // 16-byte vectors per head row
    static_assert(2 * NV <= 2 * NT, "two vectors per thread cover the key and value rows");
    AppendLoad al;
    al.slot = a.new_slots[seq];
    const size_t row = ((size_t)seq * a.num_kv_heads + kvh) * NV;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int j = (int)threadIdx.x + h * NT;
        al.x[h] = make_uint4(0, 0, 0, 0);
        if (j < 2 * NV)
            al.x[h] = reinterpret_cast<const uint4*>(j >= NV ? a.new_v : a.new_k)[row + j % NV];
    }
    return al;
}

template <typename T, int D, int BS, int NT>
__device__ __forceinline__ void append_store(const AppendLoad& al, const DecodeArgs& a, int kvh) {
    constexpr int NV = D * (int)sizeof(T) / 16;
    if (al.slot < 0) return;
    if (al.slot >= (int64_t)a.num_blocks * BS) {
        if (threadIdx.x == 0) raise_error(a.err, PA_DEVERR_SLOT);
        return;
    }
    const size_t row = ((size_t)al.slot * a.num_kv_heads + kvh) * NV;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int j = (int)threadIdx.x + h * NT;
        if (j < 2 * NV) reinterpret_cast<uint4*>(j >= NV ? a.v_cache : a.k_cache)[row + j % NV] = al.x[h];
    }
    fence_proxy_async_global();
}

// The same in one call (the cluster path), for any number of threads.
template <typename T, int D, int BS>
__device__ __forceinline__ void append_row(const DecodeArgs& a, int seq, int kvh, void* k_cache,
                                           void* v_cache) {
    constexpr int NV = D * (int)sizeof(T) / 16;          // 16-byte vectors per head row
    const int64_t slot = a.new_slots[seq];
    if (slot < 0) return;
    if (slot >= (int64_t)a.num_blocks * BS) {
        if (threadIdx.x == 0) raise_error(a.err, PA_DEVERR_SLOT);
        return;
    }
    const size_t src = ((size_t)seq * a.num_kv_heads + kvh) * NV;
    const size_t dst = ((size_t)slot * a.num_kv_heads + kvh) * NV;
    for (int i = threadIdx.x; i < 2 * NV; i += blockDim.x) {
        const bool val = i >= NV;
        const int j = val ? i - NV : i;
        const uint4 x = reinterpret_cast<const uint4*>(val ? a.new_v : a.new_k)[src + j];
        reinterpret_cast<uint4*>(val ? v_cache : k_cache)[dst + j] = x;
    }
    fence_proxy_async_global();
}

// Kernel instances: Decode = pa_decode's longest-first grid (one CTA per
// item), Cluster = pa_decode with several CTAs per item merged through
// distributed shared memory, Split = pa_decode_split's partitions, Own = the
// shared-prefix decode's own-token pass (longest-first; at head_dim 64 and
// 256 with half the warps of Decode, so that more of its CTAs fit the SMs
// beside the shared-pass CTAs -- measured faster there; at head_dim 128 the
// full-width CTA, whose shorter items win).  Each is its own instance so
// that a kernel carries only its own path's code.
enum class Mode { Decode, Cluster, Split, Own };

// ============================================================ CoreUnit ==
// fp32 FMA unit: a K/V row is spread over LPR lanes (16 bytes per lane), each
// lane forms partial dot products for all G heads of its rows, a butterfly
// reduce-scatter leaves every lane a few complete scores, probabilities go
// through a per-warp shared buffer, PV is fp32 FMA into registers.
template <typename T_, int D_, int BS_, int G_>
struct CoreUnit {
    using T = T_;
    static constexpr int D = D_, BS = BS_, G = G_;
    static constexpr int ES = (int)sizeof(T);
    static constexpr int VEC = 16 / ES;
    static constexpr int VPR = D / VEC;
    static constexpr int LPR = cmin(VPR, 32);
    static constexpr int VPL = VPR / LPR;
    static constexpr int RPP = 32 / LPR;
    static constexpr int R = cmin(BS, cmax(RPP, 4096 / (D * ES)));
    static constexpr int PASSES = R / RPP;
    static constexpr int N = PASSES * G;
    static constexpr int LOG_LPR = ilog2(LPR);
    static constexpr int RS = cmin(LOG_LPR, ilog2(N));
    static constexpr int NH = N >> RS;
    static constexpr int DUP = LPR >> RS;
    static constexpr int BOX_INNER = D;
    static constexpr int BOXES = 1;
    static constexpr int BOX_ROWS = R;            // a unit lies in one block
    static constexpr bool SWIZZLE128 = false;
    static constexpr int PBUF_FLOATS = R * G;           // per warp
    static_assert(D % VEC == 0 && VPR % LPR == 0, "head_dim must be a multiple of 16 bytes");
    static_assert(BS % R == 0 && R % RPP == 0, "unit rows must tile the block");
    static_assert((N & (N - 1)) == 0, "power-of-two score count");

    float qf[G][VPL][VEC];
    float acc[G][VPL][VEC];
    float m[G];
    float mh[NH], lh[NH];
    int hg[NH], hrow[NH];

    __device__ __forceinline__ void begin(const T* qg, float scale_log2, int lane) {
        const int c = lane % LPR, r = lane / LPR;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int v = 0; v < VPL; ++v) {
                const uint4 u = *reinterpret_cast<const uint4*>(qg + g * D + (v * LPR + c) * VEC);
                Vec16<T>::to_float(u, qf[g][v]);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    qf[g][v][e] *= scale_log2;
                    acc[g][v][e] = 0.f;
                }
            }
#pragma unroll
        for (int g = 0; g < G; ++g) m[g] = -INFINITY;
        int off = 0;
#pragma unroll
        for (int k = 0; k < RS; ++k) off += ((lane >> k) & 1) * (N >> (k + 1));
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            const int gi = j + off;
            hg[j] = gi % G;
            hrow[j] = (gi / G) * RPP + r;
            mh[j] = -INFINITY;
            lh[j] = 0.f;
        }
    }

    template <bool MASKED>
    __device__ __forceinline__ void unit(T* ks, T* vs, float* pbuf, int valid, int lane) {
        const int c = lane % LPR, r = lane / LPR;
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
        // butterfly reduce-scatter across the LPR lanes of a row
#pragma unroll
        for (int k = 0; k < RS; ++k) {
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
        for (int k = RS; k < LOG_LPR; ++k) x[0] += __shfl_xor_sync(FULL_MASK, x[0], 1 << k);

        float sc[NH];
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            sc[j] = x[j];
            if (MASKED && hrow[j] >= valid) sc[j] = -INFINITY;
        }
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
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            const float pj = exp2_approx(sc[j] - mh[j]);
            lh[j] += pj;
            pbuf[hrow[j] * G + hg[j]] = pj;
        }
        __syncwarp();
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

    __device__ __forceinline__ void drop() {
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

    // Warp partials into shared memory: wm/wl [NW][G], wacc [NW][G][D].
    __device__ __forceinline__ void publish(float* wm, float* wl, float* wacc, int warp, int lane) {
        const int c = lane % LPR, r = lane / LPR;
#pragma unroll
        for (int kk = LOG_LPR; kk < 5; ++kk)
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int v = 0; v < VPL; ++v)
#pragma unroll
                    for (int e = 0; e < VEC; ++e)
                        acc[g][v][e] += __shfl_xor_sync(FULL_MASK, acc[g][v][e], 1 << kk);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float t = 0.f;
#pragma unroll
            for (int j = 0; j < NH; ++j)
                if (hg[j] == g) t += lh[j];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) t += __shfl_xor_sync(FULL_MASK, t, off);
            if (lane == 0) {
                wm[warp * G + g] = m[g];
                wl[warp * G + g] = t * (1.0f / DUP);
            }
        }
        if (r == 0)
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int v = 0; v < VPL; ++v)
#pragma unroll
                    for (int e = 0; e < VEC; ++e)
                        wacc[(warp * G + g) * D + (v * LPR + c) * VEC + e] = acc[g][v][e];
    }
};

// ============================================================= MmaUnit ==
// Tensor-core unit for bf16: 16 tokens per unit.
//   S[16 x 16] = Q[16 x D] K^T  (rows 0..G-1 = the group's query heads,
//                               rows G..15 zero; 2 n-tiles of 8 tokens)
//   O[16 x D] += P[16 x 16] V   (P = exp2(S - m) rounded to bf16; D/8 n-tiles)
// The C fragment of the two S n-tiles is exactly the A fragment of P, so
// probabilities never leave registers.  Thread `lane` owns row g = lane / 4
// (its query head) and columns 2*(lane%4) + {0,1} of every n-tile.
// K and V tiles arrive as head_dim/64 boxes of [16 rows][128 bytes] with the
// 128-byte swizzle (16-byte chunk c of row r stored at chunk c ^ (r % 8)).
template <int D_, int BS_, int G_>
struct MmaUnit {
    using T = __nv_bfloat16;
    static constexpr int D = D_, BS = BS_, G = G_;
    static constexpr int R = 16;
    static constexpr int BOX_INNER = 64;
    static constexpr int BOXES = D / 64;
    // 8-token blocks: a unit's rows 0..7 and 8..15 come from two consecutive
    // blocks of the table, as two 8-row boxes; the second lands 1 KiB further,
    // a whole swizzle atom, so the tile's layout is that of one 16-row box
    static constexpr int BOX_ROWS = BS < R ? BS : R;
    static constexpr bool SWIZZLE128 = true;
    static constexpr int KS = D / 16;            // QK k-steps
    static constexpr int NT = D / 8;             // PV n-tiles
    static constexpr int PBUF_FLOATS = 0;
    static constexpr int BOX_BYTES = R * 128;
    static_assert(G >= 1 && G <= 8 && (BS % R == 0 || BS == 8) && D % 64 == 0, "MmaUnit shape");

    uint32_t qa[KS][2];     // A fragments of Q: row g, k-low and k-high halves
    float o[NT][2];         // PV accumulators of row g (rows 8..15 are zero padding)
    float m, l;             // row g: running max (log2 units) and this lane's partial sum
    float scale_log2;

    __device__ __forceinline__ void begin(const T* qg, float scale_log2_, int lane) {
        scale_log2 = scale_log2_;
        const int g = lane >> 2, c2 = 2 * (lane & 3);
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(qg + g * D);
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            qa[k][0] = g < G ? __ldg(qrow + (16 * k + c2) / 2) : 0u;
            qa[k][1] = g < G ? __ldg(qrow + (16 * k + 8 + c2) / 2) : 0u;
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = 0.f;
        m = -INFINITY;
        l = 0.f;
    }

    // byte offset of 16-byte chunk `chunk` (of D/8) in row `row` of a tile
    static __device__ __forceinline__ uint32_t swz(int row, int chunk) {
        return (uint32_t)((chunk >> 3) * BOX_BYTES + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
    }

    template <bool MASKED>
    __device__ __forceinline__ void unit(T* ks, T* vs, float*, int valid, int lane) {
        const uint32_t kbase = smem_addr(ks), vbase = smem_addr(vs);
        const int mi = lane >> 3, rr = lane & 7;
        // ---- S = Q K^T: ldmatrix.x4 gives both n-tiles' B fragments for one k-step
        float s0[2] = {0.f, 0.f}, s1[2] = {0.f, 0.f};
        {
            const int tok = 8 * (mi >> 1) + rr;
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                uint32_t b[4];
                ldmatrix_x4(b, kbase + swz(tok, 2 * k + (mi & 1)));
                mma_bf16_16816_top(s0[0], s0[1], qa[k][0], qa[k][1], b[0], b[1]);
                mma_bf16_16816_top(s1[0], s1[1], qa[k][0], qa[k][1], b[2], b[3]);
            }
        }
        const int c2 = 2 * (lane & 3);
        float sc[4] = {s0[0] * scale_log2, s0[1] * scale_log2, s1[0] * scale_log2,
                       s1[1] * scale_log2};
        if (MASKED) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if ((j >> 1) * 8 + c2 + (j & 1) >= valid) sc[j] = -INFINITY;
            // value rows past the end may hold NaN poison, and 0 * NaN = NaN
            uint4* vz = reinterpret_cast<uint4*>(vs);
            const int first = valid * 8, total = R * 8;        // 16-byte chunks per box
#pragma unroll
            for (int b = 0; b < BOXES; ++b)
                for (int i = first + lane; i < total; i += 32)
                    vz[b * (BOX_BYTES / 16) + i] = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async_smem();     // a later TMA load refills this stage
            __syncwarp();
        }
        // ---- lazy running max over the row's 16 scores (4 lanes x 4)
        const bool grow = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])) > m + RESCALE_THRESHOLD;
        if (__any_sync(FULL_MASK, grow)) {
            float rm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
            rm = fmaxf(rm, __shfl_xor_sync(FULL_MASK, rm, 1));
            rm = fmaxf(rm, __shfl_xor_sync(FULL_MASK, rm, 2));
            const float mn = fmaxf(m, rm);
            const float alpha = exp2_approx(m - mn);
            m = mn;
            l *= alpha;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                o[n][0] *= alpha;
                o[n][1] *= alpha;
            }
        }
        float p[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            p[j] = exp2_approx(sc[j] - m);
            l += p[j];
        }
        const uint32_t pa0 = pack_bf16x2(p[0], p[1]);     // tokens c2, c2+1
        const uint32_t pa2 = pack_bf16x2(p[2], p[3]);     // tokens 8+c2, 9+c2
        // ---- O += P V: ldmatrix.x4.trans gives B fragments of two n-tiles
        {
            const int tok = 8 * (mi & 1) + rr;
#pragma unroll
            for (int j = 0; j < NT / 2; ++j) {
                uint32_t b[4];
                ldmatrix_x4_trans(b, vbase + swz(tok, 2 * j + (mi >> 1)));
                mma_bf16_16816_top(o[2 * j][0], o[2 * j][1], pa0, pa2, b[0], b[1]);
                mma_bf16_16816_top(o[2 * j + 1][0], o[2 * j + 1][1], pa0, pa2, b[2], b[3]);
            }
        }
        __syncwarp();
    }

    __device__ __forceinline__ void drop() {
#pragma unroll
        for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = 0.f;
        m = -INFINITY;
        l = 0.f;
    }

    __device__ __forceinline__ void publish(float* wm, float* wl, float* wacc, int warp, int lane) {
        float lt = l;
        lt += __shfl_xor_sync(FULL_MASK, lt, 1);
        lt += __shfl_xor_sync(FULL_MASK, lt, 2);
        const int g = lane >> 2, c2 = 2 * (lane & 3);
        if (g < G) {
            if ((lane & 3) == 0) {
                wm[warp * G + g] = m;
                wl[warp * G + g] = lt;
            }
            float* dst = wacc + (warp * G + g) * D + c2;
#pragma unroll
            for (int n = 0; n < NT; ++n) *reinterpret_cast<float2*>(dst + 8 * n) =
                make_float2(o[n][0], o[n][1]);
        }
    }
};

// Policy choice: tensor cores for bf16 (a 16-token unit spans two 8-token
// blocks); fp32 FMAs for fp32 caches.
template <typename T, int D, int BS, int G>
using UnitFor = typename std::conditional<(std::is_same<T, __nv_bfloat16>::value &&
                                           (BS % 16 == 0 || BS == 8)),
                                          MmaUnit<D, BS, G>, CoreUnit<T, D, BS, G>>::type;

// ---------------------------------------------------- kernel geometry ----
template <class U, bool HALF_WARPS = false>
struct Layout {
    static constexpr int UNIT_BYTES = U::R * U::D * (int)sizeof(typename U::T);
    static constexpr int STAGE_BYTES = 2 * UNIT_BYTES;
    // warps per CTA: four, or two when a stage is 16 KiB (head_dim 256 on
    // the tensor-core unit), so that three CTAs still fit an SM with a
    // two-stage ring per warp (about 192 KiB of loads in flight per SM);
    // half of that for the shared-prefix decode's own-token pass at
    // head_dim 64 and 128
    static constexpr int NW = (STAGE_BYTES >= 16384 ? 2 : 4) / (HALF_WARPS ? 2 : 1);
    // stages per warp: about 12 KiB of ring per warp, at least two; with
    // 4 KiB stages (head_dim 64) the smaller CTA lets four CTAs share an SM,
    // which hides the per-CTA prologue and merge of these short items better
    static constexpr int DEPTH = cmin(8, cmax(2, 12288 / STAGE_BYTES));
    static constexpr int STAGE_REGION = NW * DEPTH * STAGE_BYTES;
    // warps merge in the drained ring: [NW][G] max, [NW][G] sum,
    // [NW][G][D] output, then the cluster exchange [G], [G], [G][D]
    static constexpr int MERGE_BYTES = (NW + 1) * U::G * (U::D + 2) * 4;
    static constexpr int MAIN_REGION = cmax(STAGE_REGION, MERGE_BYTES);
    static constexpr int PBUF_OFFSET = MAIN_REGION;
    static constexpr int ORDER_OFFSET = PBUF_OFFSET + NW * U::PBUF_FLOATS * 4;
    static constexpr int BAR_OFFSET = ORDER_OFFSET + (MAX_SORT + 4) * 4;
    // work stealing (Mode::Decode): the 16-byte cancellation response, its
    // mbarrier and the next item's index
    static constexpr int STEAL_OFFSET = (BAR_OFFSET + NW * DEPTH * 8 + 15) / 16 * 16;
    static constexpr int SMEM_BYTES = STEAL_OFFSET + 32 + 1024;   // + alignment slack
    static_assert(MAIN_REGION % 1024 == 0 && STAGE_BYTES % 1024 == 0, "1 KiB aligned stages");
    static_assert(BAR_OFFSET % 8 == 0, "mbarrier alignment");
};

// Per-CTA context shared by every item the CTA runs.
template <class U>
struct Ctx {
    unsigned char* smem;
    typename U::T* stages;     // this warp's ring
    float* pbuf;               // this warp's probability buffer (CoreUnit)
    uint64_t* bars;            // this warp's mbarriers
    int warp, lane;
    int ring;                  // units this warp has consumed so far
    int sub_blk, sub_id;       // pa_decode_step: block sub_blk of the item is sub_id (-1: none)
};

// pa_decode_step: the block of sequence seq's new token comes from its slot.
// Every CTA of the sequence reads it from there (none reads that table
// entry, so the write cannot race with a read); the CTA of kv head 0 (rank 0
// of a cluster) stores it in the table for the steps that follow.  Skipped
// sequences, slots outside the pool and empty sequences keep their entry.
template <class U>
__device__ __forceinline__ void map_new_block(Ctx<U>& cx, const DecodeArgs& a, int seq, int L,
                                              bool writer, int64_t slot) {
    cx.sub_blk = -1;
    cx.sub_id = 0;
    if (!a.table_out || L <= 0) return;
    if (slot < 0 || slot >= (int64_t)a.num_blocks * U::BS) return;
    cx.sub_blk = (L - 1) / U::BS;
    cx.sub_id = (int)(slot / U::BS);
    if (writer && threadIdx.x == 0)
        a.table_out[(size_t)seq * a.max_blocks + cx.sub_blk] = cx.sub_id;
}

// Run one item: stream this CTA's share of (seq, kvh)'s units in
// [u_begin, u_end), interleaved over `ctas` CTAs (this one is `crank`) and
// over the NW warps, then merge the warps into shared memory.  Returns with
// the CTA-merged (max, sum, unnormalised output) per (g, d) computed by
// `epilogue`.  Every thread of the CTA must call it (it holds barriers).
struct NoHook {
    __device__ void operator()() const {}
};

// `before_first` runs (on every thread) after the first window of block ids
// has been requested and before it is used: work whose loads should be in
// flight together with the window's (the fused append) goes there.
// `streamed` runs on every thread once its warp has consumed its units,
// before the warps merge (the work-stealing request goes out there, so
// that its answer arrives during the merge).
template <class U, class Ly, class Epi, class Hook = NoHook, class Hook2 = NoHook>
__device__ __forceinline__ void run_item(Ctx<U>& cx, const CUtensorMap* tm_k,
                                         const CUtensorMap* tm_v, const DecodeArgs& a, int seq,
                                         int kvh, int L, int u_begin, int u_end, int ctas,
                                         int crank, Epi&& epilogue, Hook&& before_first = Hook(),
                                         Hook2&& streamed = Hook2()) {
    using T = typename U::T;
    constexpr int NW = Ly::NW, DEPTH = Ly::DEPTH, R = U::R, D = U::D, G = U::G;
    const int warp = cx.warp, lane = cx.lane;
    const int ustride = ctas * NW;
    const int first = u_begin + crank + ctas * warp;
    const int nk = first < u_end ? (u_end - first + ustride - 1) / ustride : 0;

    const int32_t* table = a.block_tables + (size_t)seq * a.max_blocks;
    // a unit spans two 8-token blocks on the tensor-core unit with bs 8
    constexpr int HALVES = R / U::BOX_ROWS;
    static_assert(HALVES == 1 || HALVES == 2, "a unit is one box of rows or two");
    auto checked = [&](int id) {
        if (id < 0 || id >= a.num_blocks) {
            raise_error(a.err, PA_DEVERR_BLOCK_ID);
            return a.num_blocks;         // outside the tensor map: TMA fills zeros
        }
        return id;
    };
    // a window: the block ids of this warp's next 32 units, one per lane;
    // requested first, then resolved (the new token's block comes from its
    // slot under pa_decode_step, and only then is an id checked)
    int win = 0, win1 = -1, wb0 = -1;
    bool two = false;                    // the unit's second 8-token block holds tokens
    auto request_window = [&](int k0) {
        const int k = k0 + lane;
        win = 0;
        win1 = -1;
        wb0 = -1;
        two = false;
        if (k < nk) {
            const int t0 = (first + ustride * k) * R;
            wb0 = t0 / U::BS;
            win = __ldg(table + wb0);
            if constexpr (HALVES == 2) {
                two = t0 + U::BOX_ROWS < L;
                if (two) win1 = __ldg(table + wb0 + 1);
            }
        }
    };
    auto resolve_window = [&]() {
        if (wb0 < 0) {
            win = 0;
            return;
        }
        win = checked(wb0 == cx.sub_blk ? cx.sub_id : win);
        if constexpr (HALVES == 2) {
            if (two) win1 = checked(wb0 + 1 == cx.sub_blk ? cx.sub_id : win1);
        }
    };
    auto load_window = [&](int k0) {
        request_window(k0);
        resolve_window();
    };
    auto slot = [&](int k) { return (cx.ring + k) % DEPTH; };
    auto issue = [&](int k, int id, int id1) {     // lane 0 only
        const int s = slot(k);
        T* kdst = cx.stages + (size_t)s * (2 * R * D);
        const int uu = first + ustride * k;
        const int row0 = HALVES == 2 ? 0 : (uu * R) % U::BS;
        const bool second = HALVES == 2 && id1 >= 0;
        mbar_arrive_expect_tx(&cx.bars[s], (HALVES == 1 || second ? Ly::STAGE_BYTES
                                                                  : Ly::STAGE_BYTES / 2) +
                                               a.tx_extra);
#pragma unroll
        for (int b = 0; b < U::BOXES; ++b) {
            T* kb = kdst + b * R * U::BOX_INNER;
            T* vb = kdst + R * D + b * R * U::BOX_INNER;
            tma_load_4d(kb, tm_k, &cx.bars[s], b * U::BOX_INNER, kvh, row0, id);
            tma_load_4d(vb, tm_v, &cx.bars[s], b * U::BOX_INNER, kvh, row0, id);
            if (second) {
                constexpr int OFF = U::BOX_ROWS * U::BOX_INNER;
                tma_load_4d(kb + OFF, tm_k, &cx.bars[s], b * U::BOX_INNER, kvh, 0, id1);
                tma_load_4d(vb + OFF, tm_v, &cx.bars[s], b * U::BOX_INNER, kvh, 0, id1);
            }
        }
    };

    request_window(0);
    before_first();
    resolve_window();
    const int pro = cmin(DEPTH, nk);
    for (int k = 0; k < pro; ++k) {
        const int id = __shfl_sync(FULL_MASK, win, k);
        const int id1 = __shfl_sync(FULL_MASK, win1, k);
        if (lane == 0) issue(k, id, id1);
    }
    // the queries load while the first tiles are in flight
    U u;
    u.begin(reinterpret_cast<const T*>(a.q) +
                ((size_t)seq * a.num_heads + (size_t)kvh * G) * D,
            a.scale_log2, lane);
    int k = 0;
    bool failed = false;
    for (; k < nk; ++k) {
        const int s = slot(k);
        const uint32_t parity = ((cx.ring + k) / DEPTH) & 1;
        const bool landed = __all_sync(FULL_MASK, mbar_wait_bounded(&cx.bars[s], parity, a.wait_ns));
        if (!landed) {
            failed = true;
            break;
        }
        T* ks = cx.stages + (size_t)s * (2 * R * D);
        const int uu = first + ustride * k;
        const int valid = cmin(R, L - uu * R);
        if (valid == R)
            u.template unit<false>(ks, ks + R * D, cx.pbuf, valid, lane);
        else
            u.template unit<true>(ks, ks + R * D, cx.pbuf, valid, lane);
        const int kn = k + DEPTH;
        if (kn < nk) {
            if (kn % 32 == 0) load_window(kn);
            const int id = __shfl_sync(FULL_MASK, win, kn % 32);
            const int id1 = __shfl_sync(FULL_MASK, win1, kn % 32);
            if (lane == 0) issue(kn, id, id1);
        }
    }
    if (failed) {
        // A load never landed: record it, wait (bounded) for this warp's other
        // loads in flight so none lands after the CTA moves on, contribute nothing.
        if (lane == 0) raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
        const int issued = cmin(nk, k + DEPTH);
        for (int kk = k + 1; kk < issued; ++kk)
            (void)mbar_wait_bounded(&cx.bars[slot(kk)], ((cx.ring + kk) / DEPTH) & 1, a.wait_ns);
        u.drop();
        // keep the ring's phase bookkeeping consistent with what was issued
        cx.ring += issued;
    } else {
        cx.ring += nk;
    }
    streamed();                          // this thread's warp has consumed its units

    // ---- merge the warps (the merge area overlays the stage ring) ----
    __syncthreads();
    float* wm = reinterpret_cast<float*>(cx.smem);   // [NW][G]
    float* wl = wm + NW * G;                           // [NW][G]
    float* wacc = wl + NW * G;                         // [NW][G][D]
    u.publish(wm, wl, wacc, warp, lane);
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
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
        epilogue(g, d, big, num, den, wacc + NW * G * D);
    }
    // the merge area overlays the stage ring, which TMA refills next
    fence_proxy_async_smem();
}

// Whether the own-token pass of the shared-prefix decode runs half-width CTAs:
// at head_dim 64 and 128, so that more of its short items start beside the
// shared pass (three two-warp CTAs fit beside a 97 KB shared CTA at 128).  At
// 256 the shared CTA leaves no room beside it, and a two-warp CTA streams an
// item twice as fast as one warp (which took 63 of a step's 83 us).
template <class U>
__host__ __device__ constexpr bool own_half_width() { return U::D != 256; }

template <class U, Mode MODE>
__global__ void __launch_bounds__(Layout<U, MODE == Mode::Own && own_half_width<U>()>::NW * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
    using T = typename U::T;
    using Ly = Layout<U, MODE == Mode::Own && own_half_width<U>()>;
    constexpr int NW = Ly::NW, DEPTH = Ly::DEPTH, R = U::R, D = U::D, G = U::G;
    constexpr int NT = NW * 32;
    // The own-token pass of the shared-prefix decode reads nothing the
    // shared pass (the grid just before it) writes until its final merge:
    // its inputs come from grids that completed before the shared pass got
    // past its own wait.  It therefore streams its tokens first and waits for
    // the shared pass only before the merge, so the two overlap where SMs
    // are free; every CTA still waits before it leaves, which keeps the
    // stream's completion order.  pa_decode's grid stages the context
    // lengths and picks its first item before it waits: no kernel of this
    // library writes the lengths, and a caller's kernel that does completes
    // before this grid starts (it does not release its dependents early), so
    // that set-up overlaps the previous grid's last wave.  It releases its
    // own dependents only after its wait, so a grid never starts before the
    // one two launches back has completed.  Every other launch waits here.
    const bool late_wait = MODE == Mode::Own || MODE == Mode::Decode;
    if (!late_wait) pdl_wait();
    if (MODE != Mode::Decode) pdl_launch_dependents();

    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    // Split mode: a partition that does not exist leaves before anything else.
    int seq = 0, kvh = 0, L = 0, part = 0, nparts = 1;
    auto clamp_len = [&](int s) {
        int x = a.context_lens[s];
        if (x < 0 || x > a.max_tokens) {
            if (threadIdx.x == 0) raise_error(a.err, PA_DEVERR_CONTEXT_LEN);
            x = x < 0 ? 0 : a.max_tokens;
        }
        return x;
    };
    if constexpr (MODE == Mode::Split) {
        seq = blockIdx.z;
        kvh = blockIdx.y;
        part = blockIdx.x;
        L = clamp_len(seq);
        nparts = (L + a.part_tokens - 1) / a.part_tokens;
        if (part >= cmax(nparts, 1)) return;
        if (nparts > a.max_parts) {
            if (threadIdx.x == 0 && part == 0) raise_error(a.err, PA_DEVERR_WORKSPACE);
            if (part > 0) return;
            nparts = 1;                       // degrade: partition 0 covers everything
        }
        // partition 0 zeroes the reduce's arrival counts of this kv head's group
        if (part == 0 && nparts > 1 && a.ws_cnt && threadIdx.x < G)
            a.ws_cnt[(size_t)seq * a.num_heads + (size_t)kvh * G + threadIdx.x] = 0u;
    }

    Ctx<U> cx;
    cx.smem = smem;
    cx.stages = reinterpret_cast<T*>(smem) + (size_t)warp * DEPTH * (2 * R * D);
    cx.pbuf = reinterpret_cast<float*>(smem + Ly::PBUF_OFFSET) + warp * U::PBUF_FLOATS;
    cx.bars = reinterpret_cast<uint64_t*>(smem + Ly::BAR_OFFSET) + warp * DEPTH;
    cx.warp = warp;
    cx.lane = lane;
    cx.ring = 0;
    cx.sub_blk = -1;
    cx.sub_id = 0;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < DEPTH; ++s) mbar_init(&cx.bars[s], 1);
        fence_mbar_init();
        if (warp == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
        }
    }
    __syncwarp();

    T* out = reinterpret_cast<T*>(a.out);

    if constexpr (MODE == Mode::Split) {
        const int pu = a.part_tokens / R;
        const int total_units = (L + R - 1) / R;
        const int u_begin = nparts == 1 && part == 0 ? 0 : part * pu;
        const int u_end = nparts == 1 ? total_units : cmin(u_begin + pu, total_units);
        const size_t head0 = (size_t)seq * a.num_heads + (size_t)kvh * G;
        run_item<U, Ly>(cx, &tm_k, &tm_v, a, seq, kvh, L, u_begin, u_end, 1, 0,
                    [&](int g, int d, float big, float num, float den, float*) {
                        if (nparts > 1) {
                            const size_t slot = (head0 + g) * a.slot_stride + part;
                            if (d == 0) {
                                a.ws_m[slot] = big;
                                a.ws_l[slot] = den;
                            }
                            a.ws_o[slot * D + d] = num;
                        } else {
                            store_out(out + (head0 + g) * D + d, den > 0.f ? num / den : 0.f);
                        }
                    });
        return;
    } else {
        if constexpr (MODE == Mode::Cluster) {
            seq = blockIdx.z;
            kvh = blockIdx.y;
            L = clamp_len(seq);
            const int ctas = gridDim.x;
            if (a.new_slots) {
                if (blockIdx.x == 0) append_row<T, D, U::BS>(a, seq, kvh, a.k_cache, a.v_cache);
                map_new_block(cx, a, seq, L, kvh == 0 && blockIdx.x == 0, a.new_slots[seq]);
                if (ctas > 1)
                    cg::this_cluster().sync();         // every rank loads after the write
                else
                    __syncthreads();
            }
            const size_t head0 = (size_t)seq * a.num_heads + (size_t)kvh * G;
            run_item<U, Ly>(cx, &tm_k, &tm_v, a, seq, kvh, L, 0, (L + R - 1) / R, ctas, blockIdx.x,
                        [&](int g, int d, float big, float num, float den, float* x) {
                            // x: [G] max, [G] sum, [G][D] unnormalised output
                            if (ctas > 1) {
                                if (d == 0) {
                                    x[g] = big;
                                    x[G + g] = den;
                                }
                                x[2 * G + g * D + d] = num;
                            } else {
                                store_out(out + (head0 + g) * D + d, den > 0.f ? num / den : 0.f);
                            }
                        });
            if (ctas > 1) {
                float* xch = reinterpret_cast<float*>(smem) + NW * G * (D + 2);
                cg::cluster_group cluster = cg::this_cluster();
                cluster.sync();                        // every rank's xch is written
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
                cluster.sync();                        // keep xch alive until rank 0 is done
            }
            return;
        } else {
            // Which sequence sits at rank r = item / Hk of the list sorted by
            // (tokens this pass reads descending, index ascending)?  The CTA
            // stages the lengths in shared memory once.  Up to 64 sequences
            // every thread then counts, for one sequence, the entries that
            // sort before it (a direct rank: 64 compares, measured faster
            // than the search on the shared-prefix decode's own-token pass
            // and slower for 256 sequences); otherwise warp 0 selects it
            // (rank_select) from the staged values while the other warps go
            // straight to the barrier.
            const int S = a.num_seqs, Hk = a.num_kv_heads;
            // sequence, tokens this pass reads, context length, shared prefix
            int* pick = reinterpret_cast<int*>(smem + Ly::ORDER_OFFSET);
            int* lens = pick + 4;                                           // S <= MAX_SORT
            auto clamped_len = [&](int i) {
                const int x = a.context_lens[i];
                if (x < 0 || x > a.max_tokens) raise_error(a.err, PA_DEVERR_CONTEXT_LEN);
                return x < 0 ? 0 : (x > a.max_tokens ? a.max_tokens : x);
            };
            // order by the tokens this pass reads (own tokens with a shared prefix)
            auto own_tokens = [&](int i) {
                const int len = clamped_len(i);
                return len - cmin(shared_prefix_of(a, i), len);
            };
            constexpr int REG_PER_LANE = 8;
            constexpr int DIRECT_MAX = 64;
            static_assert(3 * DIRECT_MAX <= MAX_SORT, "the direct rank's arrays fit the sort area");
            constexpr int STAGED = 32 * REG_PER_LANE;
            static_assert(3 * STAGED <= MAX_SORT, "the staged lengths fit the sort area");
            const bool in_regs = S <= STAGED;
            int* own = lens;                          // up to 256: tokens this pass, length, prefix
            int* cl = lens + STAGED;
            int* pr = lens + 2 * STAGED;
            // Work stealing (pa_decode's grid): when a CTA has streamed its
            // item it asks the hardware to cancel the launch of the next CTA
            // of the grid that has not started (the next item in longest-
            // first order) and runs that item itself, until none is left.
            // The lengths are read once per CTA, and the CTA's launch, set-up
            // and length loads are not repeated per item.  Measured +2 % at
            // head_dim 128 and +3.5 % at 64 on the GQA batch; at 256, whose
            // items are twice as long, -1 %, so there each item keeps its CTA.
            constexpr bool STEAL = MODE == Mode::Decode && D <= 128;
            unsigned char* steal_answer = smem + Ly::STEAL_OFFSET;          // 16 bytes
            uint64_t* steal_bar = reinterpret_cast<uint64_t*>(steal_answer + 16);
            int* steal_next = reinterpret_cast<int*>(steal_answer + 24);
            uint32_t steal_phase = 0;
            if (STEAL && threadIdx.x == 0) {
                mbar_init(steal_bar, 1);
                fence_mbar_init();
            }
            // the lengths, once per CTA, staged in shared memory by every thread
            if (in_regs) {
                for (int i = threadIdx.x; i < S; i += NT) {
                    const int len = clamped_len(i);
                    const int p = cmin(shared_prefix_of(a, i), len);
                    own[i] = len - p;
                    cl[i] = len;
                    pr[i] = p;
                }
            } else if (S <= MAX_SORT) {
                for (int i = threadIdx.x; i < S; i += NT) lens[i] = own_tokens(i);
            }
            __syncthreads();
            bool waited = false;                            // pa_decode: griddepcontrol.wait done
            for (int item = blockIdx.x;;) {
                const int r = item / Hk;
                if (S <= DIRECT_MAX) {
                    for (int i = threadIdx.x; i < S; i += NT) {
                        const int vi = own[i];
                        int before = 0;
                        for (int k = 0; k < S; ++k) {
                            const int vk = own[k];
                            before += (vk > vi) | ((vk == vi) & (k < i));
                        }
                        if (before == r) {               // ranks are a permutation: one writer
                            pick[0] = i;
                            pick[1] = vi;
                            pick[2] = cl[i];
                            pick[3] = pr[i];
                        }
                    }
                } else if (warp == 0) {
                    int found = r, tokens = -1;                  // natural order beyond MAX_SORT
                    int len_of = 0, pre_of = 0;
                    if (in_regs) {
                        int v[REG_PER_LANE];
    #pragma unroll
                        for (int j = 0; j < REG_PER_LANE; ++j) {
                            const int i = lane + 32 * j;
                            v[j] = i < S ? own[i] : -1;
                        }
                        found = rank_select<REG_PER_LANE>([&](int j) { return v[j]; }, r, lane,
                                                          tokens);
                        len_of = cl[found];
                        pre_of = pr[found];
                    } else if (S <= MAX_SORT) {
                        found = rank_select<MAX_SORT / 32>(
                            [&](int j) {
                                const int i = lane + 32 * j;
                                return i < S ? lens[i] : -1;
                            },
                            r, lane, tokens);
                    }
                    if (lane == 0) {
                        pick[0] = found;
                        pick[1] = tokens;
                        pick[2] = len_of;
                        pick[3] = pre_of;
                    }
                }
                __syncthreads();
                seq = pick[0];
                kvh = item % Hk;
                int tok0;                                   // whole 16-token units
                if (in_regs) {
                    L = pick[2];
                    tok0 = pick[3];
                } else {
                    L = S <= MAX_SORT && !a.group_starts ? pick[1] : clamp_len(seq);
                    tok0 = cmin(shared_prefix_of(a, seq), L);
                }
                if constexpr (MODE == Mode::Decode) {
                    if (!waited) {                          // first item: see the kernel's top
                        // While the previous grid finishes, bring the tiles of
                        // each warp's first DEPTH units into L2.  The block ids
                        // are read around L1 (the grid before may still rewrite
                        // the table; the loads after the wait read it again), and
                        // a prefetch changes no data, so a stale id costs only
                        // bandwidth; ids outside the pool are skipped.
                        const int k = lane;                 // unit k of this warp
                        const int uu = tok0 / R + warp + NW * k;
                        if (k < DEPTH && uu * R < L) {
                            const int32_t* table = a.block_tables + (size_t)seq * a.max_blocks;
                            const int t0 = uu * R;
                            const int id = __ldcg(table + t0 / U::BS);
                            if (id >= 0 && id < a.num_blocks) {
                                const int row0 = U::BOX_ROWS < R ? 0 : t0 % U::BS;
#pragma unroll
                                for (int b = 0; b < U::BOXES; ++b) {
                                    tma_prefetch_l2_4d(&tm_k, b * U::BOX_INNER, kvh, row0, id);
                                    tma_prefetch_l2_4d(&tm_v, b * U::BOX_INNER, kvh, row0, id);
                                }
                            }
                        }
                        pdl_wait();
                        pdl_launch_dependents();
                        waited = true;
                    }
                }
                // the new row's loads go out here and are waited on (written,
                // fenced, barrier) only after the first window of block ids has
                // been requested, so both round trips overlap
                AppendLoad al = {};
                if (a.new_slots) al = append_load<T, D, NT>(a, seq, kvh);
                const size_t head0 = (size_t)seq * a.num_heads + (size_t)kvh * G;
                const int nchunks = a.group_starts ? (tok0 + a.chunk_tokens - 1) / a.chunk_tokens : 0;
                // x: this CTA's own part, [G] max, [G] sum, [G][D] unnormalised output,
                // kept after the exchange area when it is merged with prefix chunks
                float* x = reinterpret_cast<float*>(smem) + NW * G * (D + 2);
                run_item<U, Ly>(cx, &tm_k, &tm_v, a, seq, kvh, L, tok0 / R, (L + R - 1) / R, 1, 0,
                            [&](int g, int d, float big, float num, float den, float*) {
                                if (nchunks) {
                                    if (d == 0) {
                                        x[g] = big;
                                        x[G + g] = den;
                                    }
                                    x[2 * G + g * D + d] = num;
                                    return;
                                }
                                store_out(out + (head0 + g) * D + d, den > 0.f ? num / den : 0.f);
                            },
                            [&] {
                                if (a.new_slots) {
                                    append_store<T, D, U::BS, NT>(al, a, kvh);
                                    map_new_block(cx, a, seq, L, kvh == 0, al.slot);
                                    __syncthreads();       // the loads below see the new row
                                }
                            },
                            [&] {
                                if (STEAL && threadIdx.x == 0) {
                                    mbar_arrive_expect_tx(steal_bar, 16);
                                    clc_try_cancel(steal_answer, steal_bar);
                                }
                            });
                if constexpr (STEAL) {
                    if (threadIdx.x == 0) {
                        int next = -1;
                        if (mbar_wait_bounded(steal_bar, steal_phase, a.wait_ns))
                            next = clc_cancelled_x(steal_answer);
                        else
                            raise_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
                        *steal_next = next;
                    }
                    steal_phase ^= 1;
                    // every thread is done with the merge area (the next item's
                    // tiles land there) and reads the answer
                    __syncthreads();
                    item = *steal_next;
                    if (item < 0 || item >= (int)gridDim.x) return;
                    continue;
                }
                pdl_wait();                                // the shared pass is complete
                if (nchunks) {
                    // merge with the shared pass's chunks of each head.  A thread
                    // writes OPT groups of 4 outputs (g, d .. d+3).  It loads the
                    // maxima, sums and float4 outputs of CB chunks of every output
                    // at a time, all in flight at once (about 8 float4 per thread,
                    // which keeps them in registers at every head_dim), then
                    // rescales what it holds to the batch's new maximum and adds
                    // the batch in chunk order: one round trip per batch, and with
                    // every chunk in one batch the sums of the common maximum.
                    // The own-token pass keeps up to 16 float4 per thread in
                    // flight (4 chunks of 4 outputs at head_dim 256)
                    __syncthreads();                       // x is complete
                    constexpr int Q4 = D / 4;                        // float4 per head row
                    constexpr int OPT = (G * Q4 + NT - 1) / NT;
                    constexpr int CB = MODE == Mode::Own
                                           ? (OPT >= 16 ? 1 : OPT >= 8 ? 2 : OPT >= 4 ? 4 : 8 / OPT)
                                           : (OPT >= 8 ? 1 : 8 / OPT);    // chunks per batch
                    float mm[OPT], den[OPT];
                    float4 num[OPT];
                    int gg[OPT], qq[OPT];
    #pragma unroll
                    for (int k = 0; k < OPT; ++k) {
                        const int idx = threadIdx.x + k * NT;
                        gg[k] = idx < G * Q4 ? idx / Q4 : 0;
                        qq[k] = idx % Q4;
                        mm[k] = x[gg[k]];
                        const float* xo = x + 2 * G + gg[k] * D + 4 * qq[k];
                        num[k] = make_float4(xo[0], xo[1], xo[2], xo[3]);
                        den[k] = x[G + gg[k]];
                    }
                    auto slot_of = [&](int k, int c) {
                        return (head0 + gg[k]) * a.slot_stride + a.prefix_slot0 + c;
                    };
                    bool first = true;                     // num / den still unscaled
                    for (int c0 = 0; c0 < nchunks; c0 += CB) {
                        float bm[OPT][CB], bl[OPT][CB];
                        float4 bo[OPT][CB];
    #pragma unroll
                        for (int k = 0; k < OPT; ++k)
    #pragma unroll
                            for (int c = 0; c < CB; ++c) {
                                bm[k][c] = -INFINITY;
                                if (c0 + c < nchunks) {
                                    const size_t sl = slot_of(k, c0 + c);
                                    bm[k][c] = a.ws_m[sl];
                                    bl[k][c] = a.ws_l[sl];
                                    bo[k][c] = reinterpret_cast<const float4*>(a.ws_o + sl * D)[qq[k]];
                                }
                            }
    #pragma unroll
                        for (int k = 0; k < OPT; ++k) {
                            float nm = mm[k];
    #pragma unroll
                            for (int c = 0; c < CB; ++c) nm = fmaxf(nm, bm[k][c]);
                            // the own tokens (first batch) or the earlier batches, at nm
                            const float e0 = mm[k] == -INFINITY ? 0.f : exp2_approx(mm[k] - nm);
                            if (first || nm != mm[k]) {
                                num[k] = make_float4(e0 * num[k].x, e0 * num[k].y,
                                                     e0 * num[k].z, e0 * num[k].w);
                                den[k] = e0 * den[k];
                            }
                            mm[k] = nm;
    #pragma unroll
                            for (int c = 0; c < CB; ++c)
                                if (c0 + c < nchunks) {
                                    const float ec = exp2_approx(bm[k][c] - nm);
                                    num[k].x = fmaf(ec, bo[k][c].x, num[k].x);
                                    num[k].y = fmaf(ec, bo[k][c].y, num[k].y);
                                    num[k].z = fmaf(ec, bo[k][c].z, num[k].z);
                                    num[k].w = fmaf(ec, bo[k][c].w, num[k].w);
                                    den[k] = fmaf(ec, bl[k][c], den[k]);
                                }
                        }
                        first = false;
                    }
    #pragma unroll
                    for (int k = 0; k < OPT; ++k)
                        if (threadIdx.x + k * NT < G * Q4) {
                            T* o = out + (head0 + gg[k]) * D + 4 * qq[k];
                            const float inv = den[k] > 0.f ? 1.f / den[k] : 0.f;
                            store_out(o + 0, den[k] > 0.f ? num[k].x * inv : 0.f);
                            store_out(o + 1, den[k] > 0.f ? num[k].y * inv : 0.f);
                            store_out(o + 2, den[k] > 0.f ? num[k].z * inv : 0.f);
                            store_out(o + 3, den[k] > 0.f ? num[k].w * inv : 0.f);
                        }
                }
                return;
            }
        }
    }
}

// ---- log-sum-exp merge of split partitions ----
// grid (num_seqs * num_heads, reduce_chunks), 256 threads.  With the maximum
// M of all the head's partition maxima, chunk c sums w_p = 2^(m_p - M) times
// l_p and times o_p over its partitions: D/4 threads take the float4 columns
// of a partition's row, 256/(D/4) rows at a time (several loads in flight
// per thread), and the rows' sums fold in shared memory in a fixed order.
// With one chunk it writes the output; otherwise it leaves its sums and the
// last chunk to arrive adds them in chunk order (the result does not depend
// on the arrival order).
template <typename T, int D>
__global__ void __launch_bounds__(256) lse_reduce_kernel(const DecodeArgs a) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int NT = 256, TPR = D / 4, RP = NT / TPR;
    const int sh = blockIdx.x, chunk = blockIdx.y, C = gridDim.y;
    const int seq = sh / a.num_heads;
    int L = a.context_lens[seq];
    L = L < 0 ? 0 : cmin(L, a.max_tokens);
    const int nparts = (L + a.part_tokens - 1) / a.part_tokens;
    if (nparts <= 1 || nparts > a.max_parts) return;   // written directly by the partition kernel
    const size_t base = (size_t)sh * a.slot_stride;
    const float* m = a.ws_m + base;
    const float* l = a.ws_l + base;
    const float* o = a.ws_o + base * D;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

    __shared__ float red[NT / 32];
    __shared__ float4 rows[RP][TPR];
    __shared__ int last;
    float big = -INFINITY;
    for (int p = tid; p < nparts; p += NT) big = fmaxf(big, m[p]);
    for (int off = 16; off >= 1; off >>= 1) big = fmaxf(big, __shfl_xor_sync(FULL_MASK, big, off));
    if (lane == 0) red[warp] = big;
    __syncthreads();
    big = red[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) big = fmaxf(big, red[w]);
    __syncthreads();

    const int per = (nparts + C - 1) / C;
    const int p0 = chunk * per, p1 = cmin(nparts, p0 + per);
    float den = 0.f;
    for (int p = p0 + tid; p < p1; p += NT) den += exp2_approx(m[p] - big) * l[p];
    for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(FULL_MASK, den, off);
    if (lane == 0) red[warp] = den;
    __syncthreads();
    den = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) den += red[w];

    const int r = tid / TPR, c4 = tid % TPR;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int p = p0 + r; p < p1; p += RP) {
        const float w = exp2_approx(m[p] - big);
        const float4 v = reinterpret_cast<const float4*>(o + (size_t)p * D)[c4];
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
    }
    rows[r][c4] = acc;
    __syncthreads();
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid < TPR) {
#pragma unroll
        for (int rr = 0; rr < RP; ++rr) {
            num.x += rows[rr][tid].x;
            num.y += rows[rr][tid].y;
            num.z += rows[rr][tid].z;
            num.w += rows[rr][tid].w;
        }
    }
    T* out = reinterpret_cast<T*>(a.out) + (size_t)sh * D;
    auto write = [&](float4 n, float dd) {
        const float inv = dd > 0.f ? 1.f / dd : 0.f;
        store_out(out + 4 * tid + 0, dd > 0.f ? n.x * inv : 0.f);
        store_out(out + 4 * tid + 1, dd > 0.f ? n.y * inv : 0.f);
        store_out(out + 4 * tid + 2, dd > 0.f ? n.z * inv : 0.f);
        store_out(out + 4 * tid + 3, dd > 0.f ? n.w * inv : 0.f);
    };
    if (C == 1) {
        if (tid < TPR) write(num, den);
        return;
    }
    float* part = a.ws_part + ((size_t)sh * C + chunk) * (D + 4);
    if (tid < TPR) reinterpret_cast<float4*>(part)[tid] = num;
    if (tid == 0) part[D] = den;
    __threadfence();                                 // the sums, device-wide
    __syncthreads();
    if (tid == 0) {
        last = atomicAdd(a.ws_cnt + sh, 1u) == (unsigned)(C - 1);
        __threadfence();
    }
    __syncthreads();
    if (!last) return;
    if (tid < TPR) {
        float4 n = make_float4(0.f, 0.f, 0.f, 0.f);
        float dd = 0.f;
        for (int k = 0; k < C; ++k) {
            const float* pk = a.ws_part + ((size_t)sh * C + k) * (D + 4);
            const float4 v = __ldcg(reinterpret_cast<const float4*>(pk) + tid);
            n.x += v.x;
            n.y += v.y;
            n.z += v.z;
            n.w += v.w;
            dd += __ldcg(pk + D);
        }
        write(n, dd);
    }
    if (tid == 0) a.ws_cnt[sh] = 0;                  // ready for the next launch
}

}  // namespace pa
