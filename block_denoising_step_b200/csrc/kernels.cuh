// Memory-bound kernels of the step: coalesced 128-bit loads, warp-shuffle
// reductions, no floating-point atomics (every reduction has a fixed order).
#pragma once

#include "common.cuh"

namespace dgen {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------------ x = E[tok] (fp32 residual)
// Token ids outside [0, V) are clamped into range (never read out of bounds).
__global__ void embed_kernel(const int32_t* __restrict__ tok, const uint16_t* __restrict__ E, float* __restrict__ h,
                             int rows, int d, int V) {
    const int row = blockIdx.x;
    if (row >= rows) return;
    const int t = min(max(__ldg(&tok[row]), 0), V - 1);
    const uint4* src = reinterpret_cast<const uint4*>(E + static_cast<size_t>(t) * d);
    float4* dst = reinterpret_cast<float4*>(h + static_cast<size_t>(row) * d);
    for (int c = threadIdx.x; c < d / 8; c += blockDim.x) {
        const uint4 v = __ldg(&src[c]);
        dst[2 * c] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                                 __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
        dst[2 * c + 1] = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u),
                                     __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
    }
}

// ------------------------------------------------------------------ y = x / sqrt(mean x^2 + eps) * (1 + g) -> bf16
// One warp per row; d a multiple of 4.
__global__ void rmsnorm_kernel(const float* __restrict__ x, const uint16_t* __restrict__ g, bf16* __restrict__ y,
                               int rows, int d, float eps) {
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(row) * d);
    float ss = 0.f;
    for (int c = lane; c < d / 4; c += 32) {
        const float4 v = xr[c];
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / static_cast<float>(d) + eps);
    uint2* yr = reinterpret_cast<uint2*>(y + static_cast<size_t>(row) * d);
    const uint2* gr = reinterpret_cast<const uint2*>(g);
    for (int c = lane; c < d / 4; c += 32) {
        const float4 v = xr[c];
        const uint2 gg = __ldg(&gr[c]);
        const float g0 = 1.f + __uint_as_float(gg.x << 16), g1 = 1.f + __uint_as_float(gg.x & 0xFFFF0000u);
        const float g2 = 1.f + __uint_as_float(gg.y << 16), g3 = 1.f + __uint_as_float(gg.y & 0xFFFF0000u);
        yr[c] = make_uint2(pack2_bf16(v.x * r * g0, v.y * r * g1), pack2_bf16(v.z * r * g2, v.w * r * g3));
    }
}

// ------------------------------------------------------------------ routing permutation
// Groups the (token, slot) pairs of the top-k routing by expert, tokens in
// increasing order inside each expert (a stable counting sort), and cuts each
// expert's rows into chunks of at most `chunk` rows for the grouped GEMMs.
// One CTA of 1024 threads; E <= 256.  Deterministic: integer counts only.
constexpr int kPermTokBlock = 1024;
__global__ void __launch_bounds__(1024)
    moe_permute_kernel(const int* __restrict__ topk_id, const float* __restrict__ topk_gate, int N, int k, int E,
                       int chunk, int* __restrict__ perm_tok, float* __restrict__ perm_gate, int* __restrict__ inv,
                       int4* __restrict__ chunks, int* __restrict__ n_chunks) {
    __shared__ int s_cnt[256];
    __shared__ int s_off[256];
    __shared__ uint32_t s_sel[8][kPermTokBlock];  // bit e of token t: s_sel[e >> 5][t] >> (e & 31)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < E; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    for (int i = tid; i < N * k; i += blockDim.x) {
        const int e = __ldg(&topk_id[i]);
        if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    if (tid == 0) {
        int o = 0, nc = 0;
        for (int e = 0; e < E; ++e) {
            const int c = s_cnt[e];
            s_off[e] = o;
            for (int r = 0; r < c; r += chunk) chunks[nc++] = make_int4(e, o + r, min(chunk, c - r), 0);
            o += c;
        }
        *n_chunks = nc;
    }
    __syncthreads();
    const int words = (E + 31) >> 5;
    for (int t0 = 0; t0 < N; t0 += kPermTokBlock) {
        const int nt = min(kPermTokBlock, N - t0);
        for (int w = 0; w < words; ++w) s_sel[w][tid] = 0u;
        if (tid < nt) {
            for (int j = 0; j < k; ++j) {
                const int e = __ldg(&topk_id[static_cast<size_t>(t0 + tid) * k + j]);
                if (e >= 0 && e < E) s_sel[e >> 5][tid] |= 1u << (e & 31);
            }
        }
        __syncthreads();
        for (int e = warp; e < E; e += 32) {
            int base = s_off[e];
            for (int tt = 0; tt < nt; tt += 32) {
                const int t = tt + lane;
                const bool bit = t < nt && ((s_sel[e >> 5][t] >> (e & 31)) & 1u);
                const uint32_t mask = __ballot_sync(0xffffffffu, bit);
                if (bit) {
                    const int row = base + __popc(mask & ((1u << lane) - 1u));
                    const int token = t0 + t;
                    int j = 0;
                    while (j < k - 1 && __ldg(&topk_id[static_cast<size_t>(token) * k + j]) != e) ++j;
                    perm_tok[row] = token;
                    perm_gate[row] = __ldg(&topk_gate[static_cast<size_t>(token) * k + j]);
                    inv[static_cast<size_t>(token) * k + j] = row;
                }
                base += __popc(mask);
            }
            if (lane == 0) s_off[e] = base;
        }
        __syncthreads();
    }
}

// chunks of a dense pass over `rows` token rows (the shared FFN): {0, c*chunk, n, 0}
__global__ void dense_chunks_kernel(int rows, int chunk, int4* __restrict__ chunks, int* __restrict__ n_chunks) {
    const int nc = (rows + chunk - 1) / chunk;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) chunks[c] = make_int4(0, c * chunk, min(chunk, rows - c * chunk), 0);
    if (threadIdx.x == 0) *n_chunks = nc;
}

// dst[r][:] = src[idx[r]][:]  (bf16 rows, d a multiple of 8); one warp per row
__global__ void gather_rows_kernel(const bf16* __restrict__ src, const int* __restrict__ idx, bf16* __restrict__ dst,
                                   int n_rows, int d) {
    const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= n_rows) return;
    const int lane = threadIdx.x & 31;
    const uint4* s = reinterpret_cast<const uint4*>(src + static_cast<size_t>(__ldg(&idx[r])) * d);
    uint4* o = reinterpret_cast<uint4*>(dst + static_cast<size_t>(r) * d);
    for (int c = lane; c < d / 8; c += 32) o[c] = __ldg(&s[c]);
}

// h[t] += sum_{j<k} y[inv[t k + j]] (+ y_shared[t]), slots summed in order j = 0..k-1
__global__ void moe_combine_kernel(float* __restrict__ h, const float* __restrict__ y, const int* __restrict__ inv,
                                   const float* __restrict__ y_shared, int rows, int k, int d) {
    const int t = blockIdx.x;
    if (t >= rows) return;
    float4* hr = reinterpret_cast<float4*>(h + static_cast<size_t>(t) * d);
    for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const float4 v =
                __ldg(reinterpret_cast<const float4*>(y + static_cast<size_t>(__ldg(&inv[t * k + j])) * d) + c);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        if (y_shared) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(y_shared + static_cast<size_t>(t) * d) + c);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        float4 o = hr[c];
        o.x += acc.x;
        o.y += acc.y;
        o.z += acc.z;
        o.w += acc.w;
        hr[c] = o;
    }
}

// ------------------------------------------------------------------ softmax statistics
// (m, s, a): running max, sum of exp((L - m)/tau), first index of the max.
struct RowStat {
    float m, s;
    int a;
};

__device__ __forceinline__ RowStat stat_merge(RowStat x, RowStat y, float k) {
    RowStat r;
    r.m = fmaxf(x.m, y.m);
    const float sx = (x.m == -INFINITY) ? 0.f : x.s * exp2f((x.m - r.m) * k);
    const float sy = (y.m == -INFINITY) ? 0.f : y.s * exp2f((y.m - r.m) * k);
    r.s = sx + sy;
    r.a = (x.m > y.m || (x.m == y.m && x.a < y.a)) ? x.a : y.a;
    return r;
}

__device__ __forceinline__ RowStat warp_stat(RowStat v, float k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        RowStat w;
        w.m = __shfl_xor_sync(0xffffffffu, v.m, o);
        w.s = __shfl_xor_sync(0xffffffffu, v.s, o);
        w.a = __shfl_xor_sync(0xffffffffu, v.a, o);
        v = stat_merge(v, w, k);
    }
    return v;
}

__global__ void set_inv_tau_kernel(float* p, float inv_tau_log2) { *p = inv_tau_log2; }

// Per-(row, 256-column tile) statistics of given fp32 logits (same format as the
// LM head epilogue writes).  One warp per (row, tile).
__global__ void stats_from_logits_kernel(const float* __restrict__ logits, int rows, int V, const float* inv_tau,
                                         float* __restrict__ pmax, float* __restrict__ psum, int* __restrict__ parg) {
    const int n_tiles = V / 256;
    const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= rows * n_tiles) return;
    const int row = w / n_tiles, tile = w % n_tiles;
    const float k = __ldg(inv_tau);
    const float* src = logits + static_cast<size_t>(row) * V + tile * 256;
    RowStat st{-INFINITY, 0.f, 0};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int c = j * 32 + lane;
        const RowStat one{__ldg(&src[c]), 1.f, tile * 256 + c};
        st = stat_merge(st, one, k);
    }
    st = warp_stat(st, k);
    if (lane == 0) {
        pmax[w] = st.m;
        psum[w] = st.s;
        parg[w] = st.a;
    }
}

// Per row: merge the vocab-tile statistics -> confidence = -log(sum) (the log of
// the largest tempered probability) and the argmax.  One warp per row.
__global__ void stats_combine_kernel(const float* __restrict__ pmax, const float* __restrict__ psum,
                                     const int* __restrict__ parg, int rows, int n_tiles, const float* inv_tau,
                                     float* __restrict__ conf, int* __restrict__ argmax) {
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float k = __ldg(inv_tau);
    RowStat st{-INFINITY, 0.f, 0};
    for (int t = lane; t < n_tiles; t += 32) {
        const size_t o = static_cast<size_t>(row) * n_tiles + t;
        st = stat_merge(st, RowStat{pmax[o], psum[o], parg[o]}, k);
    }
    st = warp_stat(st, k);
    if (lane == 0) {
        conf[row] = -logf(st.s);
        argmax[row] = st.a;
    }
}

// ------------------------------------------------------------------ sampler
// One CTA per canvas, one thread per position.  Rank of an open position =
// number of open positions with larger confidence, or equal confidence and a
// lower index.  The m best are committed to their argmax and frozen; the other
// open positions are redrawn from Philox(seed; (i, s, b, 1)), lane 0.
__global__ void __launch_bounds__(1024)
    sample_commit_kernel(int32_t* __restrict__ tok, uint8_t* __restrict__ committed, const float* __restrict__ conf,
                         const int* __restrict__ argmax, int C, uint32_t V, int s, int last_step, int m_commit,
                         uint32_t k0, uint32_t k1, float* __restrict__ conf_out) {
    __shared__ float s_conf[1024];
    __shared__ uint8_t s_open[1024];
    const int b = blockIdx.x, i = threadIdx.x;
    const size_t o = static_cast<size_t>(b) * C + i;
    const bool in = i < C;
    const bool open = in && committed[o] == 0;
    const float c = in ? conf[o] : 0.f;
    s_conf[i] = c;
    s_open[i] = open ? 1 : 0;
    const int n_open = __syncthreads_count(open);
    const int m = last_step ? n_open : min(m_commit, n_open);
    if (open) {
        int rank = 0;
        for (int j = 0; j < C; ++j) {
            const float cj = s_conf[j];
            rank += (s_open[j] && (cj > c || (cj == c && j < i))) ? 1 : 0;
        }
        if (rank < m) {
            tok[o] = argmax[o];
            committed[o] = 1;
        } else {
            const Philox4 r = philox4x32_10(static_cast<uint32_t>(i), static_cast<uint32_t>(s),
                                            static_cast<uint32_t>(b), TAG_RENOISE, k0, k1);
            tok[o] = uniform_token(r.x, V);
        }
    }
    if (in && conf_out) conf_out[o] = c;
}

__global__ void init_canvas_kernel(int32_t* __restrict__ tok, uint8_t* __restrict__ committed, int B, int C,
                                   uint32_t V, uint32_t k0, uint32_t k1) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= B * C) return;
    const int b = idx / C, i = idx % C;
    const Philox4 r = philox4x32_10(static_cast<uint32_t>(i), 0u, static_cast<uint32_t>(b), TAG_INIT, k0, k1);
    tok[idx] = uniform_token(r.x, V);
    committed[idx] = 0;
}

// x_t = x0 if lane 1 < threshold (= floor(kappa 2^32)), else the uniform token of lane 0
__global__ void forward_noise_kernel(const int32_t* __restrict__ x0, int32_t* __restrict__ xt, int B, int C,
                                     uint32_t V, int step, uint64_t threshold, uint32_t k0, uint32_t k1) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= B * C) return;
    const int b = idx / C, i = idx % C;
    const Philox4 r = philox4x32_10(static_cast<uint32_t>(i), static_cast<uint32_t>(step), static_cast<uint32_t>(b),
                                    TAG_FORWARD, k0, k1);
    xt[idx] = (static_cast<uint64_t>(r.y) < threshold) ? x0[idx] : uniform_token(r.x, V);
}

}  // namespace dgen
