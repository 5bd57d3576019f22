// Routing of one MoE layer in one launch, after the router GEMM (fp32 K-split
// partials of the router logits): top-k + gates, the expert permutation with
// its chunk list, and the gather of the normed rows into expert order.
//
// Top-k gating (hyper.ai digest of the DiffusionGemma paper, model
// configuration: top-k softmax gating): the k largest router logits (larger
// first, then the lower expert id; NaN ranks below every number), gates =
// softmax over those k logits.
//
// Phase 1 (CTA b takes tokens [b TB, b TB + TB), one warp per token): lane l
// holds experts l*EPL .. l*EPL + EPL - 1 (EPL = ceil(E / 32)), each the sum of
// the n_parts partials added in part order; k rounds of a warp arg-max pick the
// top-k (or the row of `forced`, the teacher forcing of the routing in tests;
// ids of a row distinct).  The CTA counts its slots per expert in shared memory,
// marks them in a token bitmap per expert and reserves its rows of every expert
// it uses with one global atomic add per expert (tot[e]), whose return value is
// the CTA's first row inside the expert.
//
// A grid barrier follows: a counter in global memory that every CTA increments
// and waits on (bounded in time, with a growing back-off).  The counter and
// tot[] are zeroed by the pass's embedding kernel.  All CTAs are resident at
// once (grid <= SM count, small footprint).  A CTA whose wait runs out records
// ERR_ROUTE_BARRIER and leaves the consumers a state that keeps every access in
// bounds: its tokens' inverse rows point at their own slots (t k + j < rows k)
// and CTA 0 sets the chunk count to 0, so the expert GEMMs do no work and the
// combine reads rows inside its buffer.  barrier_extra (0 in normal use) raises
// the barrier's target: a test hook that makes the wait run out on purpose.
//
// Phase 2 (every CTA): the expert totals (one load per expert) give the expert
// offsets off[e] (experts in id order); a slot of token t routed to e gets row
// off[e] + (the CTA's reserved base in e) + (rank of t among this CTA's tokens
// routed to e).  Which CTA's block comes first inside an expert follows the
// order of the atomics; every row is computed independently by the grouped
// GEMMs and the combine reads rows through inv in slot order, so the results do
// not depend on it.  It writes perm_tok / perm_gate / inv and copies the
// token's normed row to xperm[row].  CTA 0 cuts each expert's rows into chunks
// of at most `chunk` rows for the grouped GEMMs, after the chunks of the shared
// FFN's pseudo-experts E .. E + n_shared - 1 over all token rows (placed first:
// the heaviest items, so the expert GEMMs take them first), the routed experts
// in id order or (kBySize) largest first, and writes the chunk count and the
// touched-expert count.  The order only decides which items the GEMMs take
// first; every chunk's rows and results are the same in any order.
//
// With E4M3 experts the gather quantizes instead of copying: each gathered row
// (and, for the shared FFN, each of the CTA's token rows in natural order) is
// written as E4M3 bytes with its power-of-two row scale (common.cuh).
//
// Every phase keeps its global loads independent of one another, so that one
// launch costs a handful of memory round trips.
#pragma once

#include "common.cuh"

namespace dgen {

constexpr int kRouteThreads = 256;
constexpr int kRouteMaxTB = 1024;    // tokens per CTA
constexpr int kRouteMaxSlots = 8192; // tokens per CTA x k
constexpr int kRouteMaxGrid = 160;   // CTAs (one routing launch; at most the SM count)
constexpr int kRouteMaxParts = 16;   // K-split partials of the router logits
constexpr int kRouteMaxEPL = 8;      // experts per lane (E <= 256)
constexpr int kRouteQuantV = 16;     // uint4 per lane in the quantizing gather (d <= 4096)

struct RouteArgs {
    const float* parts;  // [n_parts][rows][E]
    int n_parts, rows, E, k, TB;
    int* topk_id;        // [rows][k]
    float* topk_gate;
    float* logits_out;   // optional [rows][E]
    const int* forced;   // optional [rows][k]
    int chunk, n_shared;
    int* perm_tok;       // [rows k]
    float* perm_gate;
    int* inv;            // [rows][k]
    int4* chunks;
    int* n_chunks;
    int* n_touched;      // optional
    const bf16* xn;      // [rows][d]
    bf16* xperm;         // [rows k][d]
    uint8_t* xperm8;     // E4M3 experts: [rows k][d] and its row scales, instead of xperm
    float* sxperm8;
    uint8_t* xn8;        // E4M3 experts: the token rows in natural order (shared FFN) and their scales
    float* sxn8;
    int d;
    int* tot;            // [E] rows reserved per expert (zero at launch)
    unsigned int* barrier;
    unsigned int barrier_extra;  // added to the barrier target (test hook; 0 in normal use)
    int* err;
};

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// order-preserving map of a float (NaN already replaced by -inf, -0 by +0) to int
__device__ __forceinline__ int float_key(float f) {
    const int i = __float_as_int(f);
    return i >= 0 ? i : i ^ 0x7FFFFFFF;
}

__device__ __forceinline__ float key_float(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7FFFFFFF); }

// Top-k ids and gates of token `row`, computed by one warp; every lane returns
// the same ids[0..k) and gates[0..k).
__device__ __forceinline__ void route_token(const RouteArgs& a, int row, int lane, int (&ids)[kMaxTopKRouting],
                                            float (&gates)[kMaxTopKRouting]) {
    const int E = a.E, k = a.k, epl = (E + 31) / 32;
    const size_t part_stride = static_cast<size_t>(a.rows) * E;
    const float* base = a.parts + static_cast<size_t>(row) * E + lane * epl;
    float v[kRouteMaxEPL];
#pragma unroll
    for (int j = 0; j < kRouteMaxEPL; ++j) v[j] = 0.f;
    if ((epl == 4 || epl == 8) && (E & 3) == 0) {  // 16-byte loads, all partials in flight together
#pragma unroll
        for (int p = 0; p < kRouteMaxParts; ++p) {
            if (p < a.n_parts) {
#pragma unroll
                for (int c = 0; c < kRouteMaxEPL / 4; ++c) {
                    if (4 * c < epl) {
                        const float4 t = __ldg(reinterpret_cast<const float4*>(base + p * part_stride) + c);
                        v[4 * c] += t.x;
                        v[4 * c + 1] += t.y;
                        v[4 * c + 2] += t.z;
                        v[4 * c + 3] += t.w;
                    }
                }
            }
        }
    } else {
#pragma unroll
        for (int p = 0; p < kRouteMaxParts; ++p) {
            if (p < a.n_parts) {
#pragma unroll
                for (int j = 0; j < kRouteMaxEPL; ++j)
                    if (j < epl && lane * epl + j < E) v[j] += __ldg(base + p * part_stride + j);
            }
        }
    }
    int valid = 0;  // bit j: expert lane*epl + j exists
#pragma unroll
    for (int j = 0; j < kRouteMaxEPL; ++j) {
        const int e = lane * epl + j;
        if (j < epl && e < E) {
            valid |= 1 << j;
            if (a.logits_out) a.logits_out[static_cast<size_t>(row) * E + e] = v[j];
            const float x = v[j];
            v[j] = (x != x) ? -INFINITY : (x == 0.f ? 0.f : x);  // NaN lowest; -0 as +0
        }
    }
    float kept[kMaxTopKRouting];
    int taken = 0;
#pragma unroll
    for (int r = 0; r < kMaxTopKRouting; ++r) {
        if (r >= k) break;
        if (a.forced) {
            const int id = min(max(__ldg(&a.forced[static_cast<size_t>(row) * k + r]), 0), E - 1);
            const int owner = id / epl, oj = id - owner * epl;
            float mine = 0.f;
#pragma unroll
            for (int j = 0; j < kRouteMaxEPL; ++j)
                if (j == oj) mine = v[j];
            kept[r] = __shfl_sync(0xffffffffu, mine, owner);
            ids[r] = id;
            continue;
        }
        int best_key = INT_MIN, best_j = -1;
#pragma unroll
        for (int j = 0; j < kRouteMaxEPL; ++j) {
            if (((valid & ~taken) >> j) & 1) {
                const int key = float_key(v[j]);
                if (best_j < 0 || key > best_key) {
                    best_key = key;
                    best_j = j;
                }
            }
        }
        const int wmax = __reduce_max_sync(0xffffffffu, best_key);
        const unsigned int cand = __ballot_sync(0xffffffffu, best_j >= 0 && best_key == wmax);
        const int src = __ffs(cand) - 1;  // lowest lane = lowest expert ids
        const int bj = __shfl_sync(0xffffffffu, best_j, src);
        ids[r] = src * epl + bj;
        kept[r] = key_float(wmax);
        if (lane == src) taken |= 1 << bj;
    }
    float mx = -INFINITY, sum = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxTopKRouting; ++r)
        if (r < k) mx = fmaxf(mx, kept[r]);
#pragma unroll
    for (int r = 0; r < kMaxTopKRouting; ++r) {
        gates[r] = (r < k) ? expf(kept[r] - mx) : 0.f;
        sum += gates[r];
    }
    const float inv = 1.0f / sum;
#pragma unroll
    for (int r = 0; r < kMaxTopKRouting; ++r) gates[r] *= inv;
}

// Dynamic shared memory: [E][TB/32] token bitmaps, then the CTA's slots' ids,
// gates and rows ([TB k] each).
__host__ __device__ constexpr size_t route_smem_bytes(int E, int TB, int k) {
    return (static_cast<size_t>(E) * ((TB + 31) / 32) + 3 * static_cast<size_t>(TB) * k) * 4;
}

// kBySize: the routed experts' chunks largest expert first (ties by id) instead
// of in id order; a separate instantiation, so the id-order kernel carries none
// of the ranking code or its shared arrays.
template <bool kBySize>
__global__ void __launch_bounds__(kRouteThreads) moe_route_kernel(const RouteArgs a) {
    pdl_enter();
    extern __shared__ uint32_t route_sel[];
    __shared__ int s_cnt[256], s_base[256], s_off[256];
    __shared__ int s_rank[kBySize ? 256 : 1], s_cord[kBySize ? 256 : 1];  // expert -> size rank, rank -> first chunk
    __shared__ int s_ok;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, k = a.k, words = (a.TB + 31) >> 5;
    int* s_id = reinterpret_cast<int*>(route_sel + E * words);
    float* s_gate = reinterpret_cast<float*>(s_id + a.TB * k);
    int* s_row = reinterpret_cast<int*>(s_gate + a.TB * k);
    const int t0 = blockIdx.x * a.TB, nt = max(0, min(a.TB, a.rows - t0));
    for (int i = tid; i < E * words; i += kRouteThreads) route_sel[i] = 0u;
    for (int e = tid; e < 256; e += kRouteThreads) s_cnt[e] = 0;
    __syncthreads();

    // phase 1: top-k and gates of this CTA's tokens
    for (int lt = warp; lt < nt; lt += kRouteThreads / 32) {
        const int row = t0 + lt;
        int ids[kMaxTopKRouting];
        float gates[kMaxTopKRouting];
        route_token(a, row, lane, ids, gates);
        if (lane < k) {
            int id = 0;
            float gt = 0.f;
#pragma unroll
            for (int r = 0; r < kMaxTopKRouting; ++r)
                if (r == lane) {
                    id = ids[r];
                    gt = gates[r];
                }
            a.topk_id[static_cast<size_t>(row) * k + lane] = id;
            a.topk_gate[static_cast<size_t>(row) * k + lane] = gt;
            s_id[lt * k + lane] = id;
            s_gate[lt * k + lane] = gt;
            atomicAdd(&s_cnt[id], 1);
            atomicOr(&route_sel[id * words + (lt >> 5)], 1u << (lt & 31));
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouteThreads) s_base[e] = s_cnt[e] ? atomicAdd(&a.tot[e], s_cnt[e]) : 0;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        int ok = 1;
        atomicAdd(a.barrier, 1u);
        // poll with a growing back-off: many CTAs polling one L2 line would slow
        // the very atomics they wait for
        const uint64_t start = globaltimer_ns();
        uint32_t nap = 32;
        const unsigned int target = gridDim.x + a.barrier_extra;
        for (uint32_t i = 1; ld_acquire_u32(a.barrier) < target; ++i) {
            if ((i & 15u) == 0 && globaltimer_ns() - start > kWaitLimitNs) {
                atomicExch(a.err, ERR_ROUTE_BARRIER);
                ok = 0;
                break;
            }
            __nanosleep(nap);
            nap = min(nap * 2, 1024u);
        }
        s_ok = ok;
    }
    __syncthreads();
    if (!s_ok) {  // safe state for the consumers (see the header comment)
        for (int i = tid; i < nt * k; i += kRouteThreads) a.inv[static_cast<size_t>(t0) * k + i] = t0 * k + i;
        if (blockIdx.x == 0 && tid == 0) *a.n_chunks = 0;
        return;
    }

    // phase 2: expert totals -> offsets (and, in CTA 0, the chunk list)
    for (int e = tid; e < E; e += kRouteThreads) s_cnt[e] = __ldcg(&a.tot[e]);
    __syncthreads();
    const bool by_size = kBySize && blockIdx.x == 0;  // the same for the whole CTA
    if (by_size) {  // rank of each expert by row count, largest first, ties by id (a permutation)
        for (int e = tid; e < E; e += kRouteThreads) {
            const int c = s_cnt[e];
            int r = 0;
            for (int f = 0; f < E; ++f) {
                const int cf = s_cnt[f];
                r += (cf > c) || (cf == c && f < e);
            }
            s_rank[e] = r;
            s_cord[r] = (c + a.chunk - 1) / a.chunk;
        }
        __syncthreads();
    }
    if (warp == 0) {  // exclusive scans of the row and chunk counts; lane owns experts 8 lane .. 8 lane + 7
        int cnt[8], nch[8], tot = 0, totc = 0, used = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            cnt[j] = e < E ? s_cnt[e] : 0;
            nch[j] = (cnt[j] + a.chunk - 1) / a.chunk;
            tot += cnt[j];
            totc += nch[j];
            used += cnt[j] > 0;
        }
        int inc = tot, incc = totc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o), yc = __shfl_up_sync(0xffffffffu, incc, o);
            if (lane >= o) {
                inc += y;
                incc += yc;
            }
        }
        // the shared FFN's chunks come first (the heaviest items: all token rows of
        // a slice), the routed experts' after them
        const int per = (a.rows + a.chunk - 1) / a.chunk;
        const int n_sh_chunks = a.n_shared * per;
        int base = inc - tot, cbase = n_sh_chunks + incc - totc;
        const bool lead = blockIdx.x == 0;
        if (by_size) {  // first chunk of each rank: exclusive scan in rank order, lane owns ranks 8 lane ..
            int nr[8], totr = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                nr[j] = lane * 8 + j < E ? s_cord[lane * 8 + j] : 0;
                totr += nr[j];
            }
            int incr = totr;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incr, o);
                if (lane >= o) incr += y;
            }
            int start = n_sh_chunks + incr - totr;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (lane * 8 + j < E) s_cord[lane * 8 + j] = start;
                start += nr[j];
            }
            __syncwarp();
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            if (e < E) {
                s_off[e] = base;
                if (lead) {
                    const int cb = by_size ? s_cord[s_rank[e]] : cbase;
                    for (int r = 0; r < nch[j]; ++r)
                        a.chunks[cb + r] = make_int4(e, base + r * a.chunk, min(a.chunk, cnt[j] - r * a.chunk), 0);
                }
                base += cnt[j];
                cbase += nch[j];
            }
        }
        if (lead) {
            used = __reduce_add_sync(0xffffffffu, used);
            if (lane == 0 && a.n_touched) *a.n_touched = used;  // experts routed to (whose weights are read)
            const int routed = __shfl_sync(0xffffffffu, incc, 31);
            for (int i = lane; i < n_sh_chunks; i += 32) {
                const int j = i / per, r = i - j * per;
                a.chunks[i] = make_int4(E + j, r * a.chunk, min(a.chunk, a.rows - r * a.chunk), 0);
            }
            if (lane == 31) *a.n_chunks = routed + n_sh_chunks;
        }
    }
    __syncthreads();
    // rows of this CTA's slots
    for (int i = tid; i < nt * k; i += kRouteThreads) {
        const int lt = i / k, t = t0 + lt;
        const int e = s_id[i];
        const uint32_t* sel = route_sel + e * words;
        int rank = 0;
        for (int w = 0; w < (lt >> 5); ++w) rank += __popc(sel[w]);
        rank += __popc(sel[lt >> 5] & ((1u << (lt & 31)) - 1u));
        const int row = s_off[e] + s_base[e] + rank;
        a.perm_tok[row] = t;
        a.perm_gate[row] = s_gate[i];
        a.inv[static_cast<size_t>(t0) * k + i] = row;
        s_row[i] = row;
    }
    __syncthreads();
    const int d8 = a.d / 8;
    if (a.xperm8) {
        // quantizing gather: xperm8[row] = E4M3(xn[token]), one warp per slot, then
        // the CTA's own token rows in natural order (one warp per token)
        for (int i = warp; i < nt * k + nt; i += kRouteThreads / 32) {
            const bool slot = i < nt * k;
            const int t = slot ? t0 + i / k : t0 + (i - nt * k);
            const uint4* src = reinterpret_cast<const uint4*>(a.xn + static_cast<size_t>(t) * a.d);
            uint4 v[kRouteQuantV];
            float amax = 0.f;
#pragma unroll
            for (int j = 0; j < kRouteQuantV; ++j) {
                const int c = lane + 32 * j;
                v[j] = c < d8 ? __ldg(&src[c]) : make_uint4(0, 0, 0, 0);
                amax = fmaxf(amax, bf16x8_absmax(v[j]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            float sc, inv;
            e4m3_row_scale(amax, sc, inv);
            const size_t r = slot ? static_cast<size_t>(s_row[i]) : static_cast<size_t>(t);
            uint2* dst = reinterpret_cast<uint2*>((slot ? a.xperm8 : a.xn8) + r * a.d);
#pragma unroll
            for (int j = 0; j < kRouteQuantV; ++j) {
                const int c = lane + 32 * j;
                if (c < d8) dst[c] = bf16x8_to_e4m3(v[j], inv);
            }
            if (lane == 0) (slot ? a.sxperm8 : a.sxn8)[r] = sc;
        }
        return;
    }
    // gather: xperm[row] = xn[token], one warp per two slots, each row's loads all
    // in flight before its stores (one memory round trip per pair of rows)
    constexpr int kGatherSlots = 2;
    for (int i0 = warp * kGatherSlots; i0 < nt * k; i0 += (kRouteThreads / 32) * kGatherSlots) {
        uint4 v[kGatherSlots][kRouteQuantV];
#pragma unroll
        for (int u = 0; u < kGatherSlots; ++u) {
            const int i = i0 + u;
            const uint4* src = reinterpret_cast<const uint4*>(a.xn + static_cast<size_t>(t0 + min(i, nt * k - 1) / k) * a.d);
#pragma unroll
            for (int j = 0; j < kRouteQuantV; ++j) {
                const int c = lane + 32 * j;
                v[u][j] = (i < nt * k && c < d8) ? __ldg(&src[c]) : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < kGatherSlots; ++u) {
            const int i = i0 + u;
            if (i >= nt * k) break;
            uint4* dst = reinterpret_cast<uint4*>(a.xperm + static_cast<size_t>(s_row[i]) * a.d);
#pragma unroll
            for (int j = 0; j < kRouteQuantV; ++j) {
                const int c = lane + 32 * j;
                if (c < d8) dst[c] = v[u][j];
            }
        }
    }
}

}  // namespace dgen
