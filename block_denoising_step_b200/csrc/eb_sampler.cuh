// The pages' own sampler (hyper.ai digest of the DiffusionGemma paper, Method,
// sampler paragraph and adaptive stopping): entropy-bounded acceptance with
// adaptive stopping, on the LM head's per-tile statistics or on given fp32 logits.
//
// eb_stats_combine_kernel: one warp per canvas row merges the LM-head
// epilogue's per-(row, vocab tile) (max, S, T, argmax) into the row's entropy
// H = ln S - ln 2 T / S and argmax (no stored logits).
//
// entropy_row_kernel: one 256-thread block per canvas row reduces the row's V
// logits to (running max M, s = sum 2^((L - M) k), t = sum 2^((L - M) k) (L - M) k,
// argmax) with k = log2(e) / tau, then H = ln s - ln 2 * t / s (nats), the
// entropy of Softmax(L / tau).
//
// eb_commit_kernel: one block per canvas, one thread per position.  Open
// positions (with freeze = 0: every position, so earlier choices can be revised)
// rank by (entropy, position); the sorted entropies' exclusive prefix
// sums bound the mutual information of each prefix (entropy-bounded unmasking:
// sum - max over an ascending prefix = sum of all but its last); the first
// prefix position whose bound reaches gamma is rejected with everything after
// it (the first position is always accepted).  Accepted positions commit to
// their argmax and freeze; the others are redrawn from Philox(seed; (i, s, b, 1)).
// Stop test (after a step of a block, s > 0): mean entropy over the canvas
// below stop_threshold and every argmax equal to the previous step's; on a stop,
// and on the last step of the budget, every open position commits to its argmax.
// A canvas that has stopped (or, frozen, has every position committed) is done:
// later steps of the same block leave it unchanged (done[] is cleared at s = 0).
#pragma once

#include "common.cuh"

namespace dgen {

struct EntStat {
    float m, s, t;
    int a;
};

__device__ __forceinline__ EntStat ent_merge(EntStat x, EntStat y, float k) {
    if (y.m == -INFINITY) return x;
    if (x.m == -INFINITY) return y;
    EntStat r;
    r.m = fmaxf(x.m, y.m);
    const float dx = (x.m - r.m) * k, dy = (y.m - r.m) * k;  // <= 0, log2 units
    const float fx = exp2f(dx), fy = exp2f(dy);
    r.s = x.s * fx + y.s * fy;
    r.t = fx * (x.t + x.s * dx) + fy * (y.t + y.s * dy);
    r.a = (x.m > y.m || (x.m == y.m && x.a < y.a)) ? x.a : y.a;
    return r;
}

__global__ void __launch_bounds__(256) entropy_row_kernel(const float* __restrict__ logits, int rows, int V,
                                                          const float* __restrict__ inv_tau_log2,
                                                          float* __restrict__ entropy, int* __restrict__ argmax) {
    pdl_enter();
    __shared__ EntStat red[8];
    const int row = blockIdx.x;
    if (row >= rows) return;
    const float k = __ldg(inv_tau_log2);
    const float4* src = reinterpret_cast<const float4*>(logits + static_cast<size_t>(row) * V);
    EntStat st{-INFINITY, 0.f, 0.f, 0};
    for (int c = threadIdx.x; c < V / 4; c += 256) {  // column order within a thread: ascending
        const float4 q = __ldg(&src[c]);
        const float xs[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) st = ent_merge(st, EntStat{xs[e], 1.f, 0.f, 4 * c + e}, k);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        EntStat w;
        w.m = __shfl_xor_sync(0xffffffffu, st.m, o);
        w.s = __shfl_xor_sync(0xffffffffu, st.s, o);
        w.t = __shfl_xor_sync(0xffffffffu, st.t, o);
        w.a = __shfl_xor_sync(0xffffffffu, st.a, o);
        st = ent_merge(st, w, k);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = st;
    __syncthreads();
    if (threadIdx.x == 0) {
        EntStat r = red[0];
        for (int w = 1; w < 8; ++w) r = ent_merge(r, red[w], k);
        entropy[row] = logf(r.s) - 0.69314718055994531f * r.t / r.s;
        argmax[row] = r.a;
    }
}

// Per row: merge the LM head's per-tile statistics (max, S, T, argmax; T in
// log2 units relative to the tile max) into the entropy and argmax.  One warp per row.
__global__ void eb_stats_combine_kernel(const float* __restrict__ pmax, const float* __restrict__ psum,
                                        const float* __restrict__ pent, const int* __restrict__ parg, int rows,
                                        int n_tiles, const float* __restrict__ inv_tau_log2,
                                        float* __restrict__ entropy, int* __restrict__ argmax) {
    pdl_enter();
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float k = __ldg(inv_tau_log2);
    EntStat st{-INFINITY, 0.f, 0.f, 0};
    for (int t = lane; t < n_tiles; t += 32) {  // tiles in ascending order within a lane
        const size_t o = static_cast<size_t>(row) * n_tiles + t;
        st = ent_merge(st, EntStat{pmax[o], psum[o], pent[o], parg[o]}, k);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        EntStat w;
        w.m = __shfl_xor_sync(0xffffffffu, st.m, o);
        w.s = __shfl_xor_sync(0xffffffffu, st.s, o);
        w.t = __shfl_xor_sync(0xffffffffu, st.t, o);
        w.a = __shfl_xor_sync(0xffffffffu, st.a, o);
        st = ent_merge(st, w, k);
    }
    if (lane == 0) {
        entropy[row] = logf(st.s) - 0.69314718055994531f * st.t / st.s;
        argmax[row] = st.a;
    }
}

__global__ void __launch_bounds__(1024)
    eb_commit_kernel(int32_t* __restrict__ tok, uint8_t* __restrict__ committed, const float* __restrict__ entropy,
                     const int* __restrict__ argmax, int* __restrict__ prev_argmax, uint8_t* __restrict__ done,
                     int C, uint32_t V, int s, int last_step, int freeze, float gamma, float stop_threshold,
                     uint32_t pos_off, uint32_t k0, uint32_t k1, uint8_t* __restrict__ stop_out) {
    pdl_enter();
    __shared__ float s_h[1024];
    __shared__ uint8_t s_open[1024];
    __shared__ float s_sorted[1024];
    __shared__ float s_red[32];
    __shared__ int s_first_reject;
    const int b = blockIdx.x, i = threadIdx.x;
    const size_t o = static_cast<size_t>(b) * C + i;
    const bool in = i < C;
    if (s > 0 && done[b]) {  // finished earlier in this block: unchanged
        if (i == 0 && stop_out) stop_out[b] = 1;
        return;
    }
    const bool open = in && (!freeze || committed[o] == 0);
    const float h = in ? entropy[o] : 0.f;
    const int am = in ? argmax[o] : 0;
    s_h[i] = h;
    s_open[i] = open ? 1 : 0;
    if (i == 0) s_first_reject = 0x7fffffff;
    // stop test: mean entropy (block sum in a fixed order) and an unchanged argmax canvas
    float v = h;
#pragma unroll
    for (int w = 16; w > 0; w >>= 1) v += __shfl_xor_sync(0xffffffffu, v, w);
    if ((i & 31) == 0) s_red[i >> 5] = v;
    const int same = __syncthreads_and(!in || s <= 0 || prev_argmax[o] == am);
    float total = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) total += s_red[w];
    const bool stop = s > 0 && same && total / static_cast<float>(C) < stop_threshold;
    const int n_open = __syncthreads_count(open);
    // rank of an open position among the open ones by (entropy, position)
    int rank = 0;
    if (open) {
        for (int j = 0; j < C; ++j) {
            const float hj = s_h[j];
            rank += (s_open[j] && (hj < h || (hj == h && j < i))) ? 1 : 0;
        }
        s_sorted[rank] = h;
    }
    __syncthreads();
    // exclusive prefix sum of the sorted entropies, in rank order (one thread)
    if (i == 0) {
        float acc = 0.f;
        for (int r = 0; r < n_open; ++r) {
            if (r > 0 && acc >= gamma) {
                s_first_reject = r;
                break;
            }
            acc += s_sorted[r];
        }
    }
    __syncthreads();
    const int k_accept = (last_step || stop) ? n_open : min(n_open, s_first_reject);
    if (open) {
        if (rank < k_accept) {
            tok[o] = am;
            committed[o] = 1;
        } else {
            const Philox4 r = philox4x32_10(pos_off + static_cast<uint32_t>(i), static_cast<uint32_t>(s),
                                            static_cast<uint32_t>(b), TAG_RENOISE, k0, k1);
            tok[o] = uniform_token(r.x, V);
            committed[o] = 0;
        }
    }
    if (in) prev_argmax[o] = am;
    // done: stopped, or (frozen) nothing left open
    const int n_acc = __syncthreads_count(open && rank < k_accept);
    if (i == 0) {
        done[b] = (stop || last_step || (freeze && n_acc == n_open)) ? 1 : 0;
        if (stop_out) stop_out[b] = stop ? 1 : 0;
    }
}

}  // namespace dgen
