// Memory-bound kernels of the step: coalesced 128-bit loads, warp-shuffle
// reductions, no floating-point atomics (every reduction has a fixed order).
#pragma once

#include "common.cuh"

namespace dgen {

constexpr int kMaxTopKRouting = 16;

}  // namespace dgen

#include "routing.cuh"

namespace dgen {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Block-wide sum (blockDim.x a multiple of 32, at most 256), same order on every call.
__device__ __forceinline__ float block_sum(float v, float* red) {
    v = warp_sum(v);
    const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    float t = 0.f;
    for (int i = 0; i < nw; ++i) t += red[i];
    return t;
}

// Writes y = x / sqrt(mean x^2 + eps) * (1 + g) as bf16 for a row held as
// float4 values v[i] at columns 4 (threadIdx.x + blockDim.x i).
template <int MAXV>
__device__ __forceinline__ void norm_row_store(const float4 (&v)[MAXV], int d4, const uint16_t* __restrict__ g,
                                               bf16* __restrict__ y, float eps, float* red) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int c = threadIdx.x + blockDim.x * i;
        if (c < d4) ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / static_cast<float>(4 * d4) + eps);
    const uint2* gr = reinterpret_cast<const uint2*>(g);
    uint2* yr = reinterpret_cast<uint2*>(y);
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int c = threadIdx.x + blockDim.x * i;
        if (c < d4) {
            const uint2 gg = __ldg(&gr[c]);
            const float g0 = 1.f + __uint_as_float(gg.x << 16), g1 = 1.f + __uint_as_float(gg.x & 0xFFFF0000u);
            const float g2 = 1.f + __uint_as_float(gg.y << 16), g3 = 1.f + __uint_as_float(gg.y & 0xFFFF0000u);
            yr[c] = make_uint2(pack2_bf16(v[i].x * r * g0, v[i].y * r * g1), pack2_bf16(v[i].z * r * g2, v[i].w * r * g3));
        }
    }
}

constexpr int kRowMaxV = 8;  // 128 threads x 8 float4: rows up to d = 4096
constexpr int kMaxParts = 8;  // K-split partials / shared-FFN slices summed by the row kernels
constexpr int kMaxScSplits = 32;  // K-split partials of the self-conditioning p0_hat E GEMM

// Row kernels below run one block per token row with kRowCols float4 columns
// per thread (columns threadIdx.x + blockDim.x * i): blockDim = d / 8 rounded up
// to a warp (d <= 4096), small enough that several rows' blocks share an SM,
// while every source row's loads of a thread are in flight together.
constexpr int kRowCols = 2;  // float4 columns per thread in the row kernels
constexpr int kCombineSlots = 8;   // expert slots the one-round-trip combine holds (top_k <= 8)
constexpr int kCombineShared = 4;  // shared-FFN slices it holds
constexpr int kResidParts = 4;     // K-split partials the residual kernel loads in its first round
__host__ __device__ constexpr int row_threads(int d) { return ((d / 4 + kRowCols - 1) / kRowCols + 31) / 32 * 32; }

// ------------------------------------------------------------------ residual add of K-split partials + norm
// h[t] += sum_{s < n_parts} parts[s][t] (split order), then y[t] = RMSNorm(h[t])
// with gain g.
__global__ void __launch_bounds__(512) residual_norm_kernel(float* __restrict__ h, const float* __restrict__ parts,
                                                            int n_parts, size_t part_stride, int rows, int d,
                                                            const uint16_t* __restrict__ g, bf16* __restrict__ y,
                                                            float eps) {
    pdl_enter();
    __shared__ float red[32];
    const int t = blockIdx.x;
    if (t >= rows) return;
    const int d4 = d / 4;
    float4* hr = reinterpret_cast<float4*>(h + static_cast<size_t>(t) * d);
    // every partial and h of both columns loaded before the sums (one round trip)
    float4 q[kRowCols][kResidParts + 1];
#pragma unroll
    for (int i = 0; i < kRowCols; ++i) {
        const int c = threadIdx.x + blockDim.x * i;
        const bool in = c < d4;
#pragma unroll
        for (int sp = 0; sp < kResidParts; ++sp)
            q[i][sp] = (in && sp < n_parts)
                           ? __ldg(reinterpret_cast<const float4*>(parts + sp * part_stride + static_cast<size_t>(t) * d) + c)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        q[i][kResidParts] = in ? hr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // partials beyond kResidParts (not used by the path's split choices) in a second round
    float4 v[kRowCols];
#pragma unroll
    for (int i = 0; i < kRowCols; ++i) {
        const int c = threadIdx.x + blockDim.x * i;
        float4 o = q[i][kResidParts];
#pragma unroll
        for (int sp = 0; sp < kResidParts; ++sp) {
            o.x += q[i][sp].x;
            o.y += q[i][sp].y;
            o.z += q[i][sp].z;
            o.w += q[i][sp].w;
        }
        for (int sp = kResidParts; sp < n_parts; ++sp) {
            if (c >= d4) break;
            const float4 a = __ldg(reinterpret_cast<const float4*>(parts + sp * part_stride + static_cast<size_t>(t) * d) + c);
            o.x += a.x;
            o.y += a.y;
            o.z += a.z;
            o.w += a.w;
        }
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c < d4) {
            hr[c] = o;
            v[i] = o;
        }
    }
    norm_row_store<kRowCols>(v, d4, g, y + static_cast<size_t>(t) * d, eps, red);
}

// ------------------------------------------------------------------ QKV partials -> RoPE -> q / KV cache
// Sums the K-split partials of the packed projection (q heads, k heads, v
// heads of hd features), rotates q and k (rotate-half pairs (j, j + hd/2) by
// pos * base^(-2j/hd), cos/sin from the table) and writes bf16 q [B][Hq][n_q][hd]
// and the K / V cache [B][Hkv][S_max][hd] at position pos0 + i.  One block of
// hd/2 threads per (row, head).
__global__ void rope_scatter_kernel(const float* __restrict__ parts, int n_parts, size_t part_stride, int rows,
                                    int n_q, int pos0, int Hq, int Hkv, int hd, int S_max,
                                    const float2* __restrict__ rope, bf16* __restrict__ q_out,
                                    bf16* __restrict__ k_cache, bf16* __restrict__ v_cache) {
    pdl_enter();
    const int row = blockIdx.x, head = blockIdx.y, j = threadIdx.x, half = hd >> 1;
    if (row >= rows) return;
    const int b = row / n_q, i = row - b * n_q, pos = pos0 + i;
    const int width = (Hq + 2 * Hkv) * hd;
    const float* src = parts + static_cast<size_t>(row) * width + head * hd;
    float x1 = 0.f, x2 = 0.f;
    for (int sp = 0; sp < n_parts; ++sp) {
        x1 += __ldg(&src[sp * part_stride + j]);
        x2 += __ldg(&src[sp * part_stride + j + half]);
    }
    bf16* dst;
    if (head < Hq) {
        dst = q_out + ((static_cast<size_t>(b) * Hq + head) * n_q + i) * hd;
    } else if (head < Hq + Hkv) {
        dst = k_cache + ((static_cast<size_t>(b) * Hkv + (head - Hq)) * S_max + pos) * hd;
    } else {
        dst = v_cache + ((static_cast<size_t>(b) * Hkv + (head - Hq - Hkv)) * S_max + pos) * hd;
    }
    if (head < Hq + Hkv) {
        const float2 cs = __ldg(&rope[static_cast<size_t>(pos) * half + j]);
        const float a = x1 * cs.x - x2 * cs.y, c = x2 * cs.x + x1 * cs.y;
        x1 = a;
        x2 = c;
    }
    dst[j] = __float2bfloat16_rn(x1);
    dst[j + half] = __float2bfloat16_rn(x2);
}


// x = E[tok] (fp32 residual) and, fused, y = RMSNorm(x) with gain g (the first
// layer's attention norm).  One 128-thread block per row.
// With z set (self-conditioning) x = E[tok] + z, z the sum of its z_parts
// K-split partials in split order.
__global__ void __launch_bounds__(128) embed_norm_kernel(const int32_t* __restrict__ tok, const uint16_t* __restrict__ E,
                                                         float* __restrict__ h, const uint16_t* __restrict__ g,
                                                         bf16* __restrict__ y, int rows, int d, int V, float eps,
                                                         unsigned int* __restrict__ zero_words, int n_zero,
                                                         const float* __restrict__ z, int z_parts, size_t z_stride) {
    pdl_enter();
    if (blockIdx.x == 0)  // the pass's grid-barrier counters
        for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero_words[i] = 0u;
    __shared__ float red[4];
    const int row = blockIdx.x;
    if (row >= rows) return;
    const int t = min(max(__ldg(&tok[row]), 0), V - 1);
    const uint2* src = reinterpret_cast<const uint2*>(E + static_cast<size_t>(t) * d);
    float4* hr = reinterpret_cast<float4*>(h + static_cast<size_t>(row) * d);
    const int d4 = d / 4;
    float4 v[kRowMaxV];
#pragma unroll
    for (int i = 0; i < kRowMaxV; ++i) {
        const int c = threadIdx.x + 128 * i;
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c < d4) {
            const uint2 e = __ldg(&src[c]);
            v[i] = make_float4(__uint_as_float(e.x << 16), __uint_as_float(e.x & 0xFFFF0000u),
                               __uint_as_float(e.y << 16), __uint_as_float(e.y & 0xFFFF0000u));
            if (z) {
                const float4* zr = reinterpret_cast<const float4*>(z + static_cast<size_t>(row) * d) + c;
                float4 zs = zr[0];
                for (int s = 1; s < z_parts; ++s) {
                    const float4 a = zr[s * (z_stride / 4)];
                    zs.x += a.x;
                    zs.y += a.y;
                    zs.z += a.z;
                    zs.w += a.w;
                }
                v[i].x += zs.x;
                v[i].y += zs.y;
                v[i].z += zs.z;
                v[i].w += zs.w;
            }
            hr[c] = v[i];
        }
    }
    norm_row_store<kRowMaxV>(v, d4, g, y + static_cast<size_t>(row) * d, eps, red);
}

// h[t] += sum_{s<y_splits} sum_{j<k} y[s][inv[t k + j]] + sum_{j<n_shared} y_shared[j][t]:
// the terms summed in that order (K-split partials outermost, slots j = 0..k-1,
// then the shared FFN's feature-slice parts) and added to h; then, if g is not
// null, the next normed input y_norm[t] = RMSNorm(h[t]) with gain g (fused).
// With one split, at most kCombineSlots slots and kCombineShared slices (every
// workload here) all of a thread's loads are in flight before the first sum.
__global__ void __launch_bounds__(512) moe_combine_norm_kernel(float* __restrict__ h, const float* __restrict__ y,
                                                               size_t y_split_stride, int y_splits,
                                                               const int* __restrict__ inv,
                                                               const float* __restrict__ y_shared, int n_shared,
                                                               int rows, int k, int d, const uint16_t* __restrict__ g,
                                                               bf16* __restrict__ y_norm, float eps) {
    pdl_enter();
    __shared__ float red[32];
    __shared__ int s_r[kMaxTopKRouting];
    const int t = blockIdx.x;
    if (t >= rows) return;
    if (threadIdx.x < k) s_r[threadIdx.x] = __ldg(&inv[t * k + threadIdx.x]);
    __syncthreads();
    const int d4 = d / 4;
    float4* hr = reinterpret_cast<float4*>(h + static_cast<size_t>(t) * d);
    float4 v[kRowCols];
    if (y_splits == 1 && k <= kCombineSlots && n_shared <= kCombineShared) {
        // every source row's loads of both columns are issued before any sum:
        // one memory round trip for the whole row
        float4 q[kRowCols][kCombineSlots + kCombineShared + 1];
#pragma unroll
        for (int i = 0; i < kRowCols; ++i) {
            const int c = threadIdx.x + blockDim.x * i;
            const bool in = c < d4;
#pragma unroll
            for (int j = 0; j < kCombineSlots; ++j)
                q[i][j] = (in && j < k) ? __ldg(reinterpret_cast<const float4*>(y + static_cast<size_t>(s_r[j]) * d) + c)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < kCombineShared; ++j)
                q[i][kCombineSlots + j] =
                    (in && j < n_shared)
                        ? __ldg(reinterpret_cast<const float4*>(y_shared + (static_cast<size_t>(j) * rows + t) * d) + c)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
            q[i][kCombineSlots + kCombineShared] = in ? hr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kRowCols; ++i) {
            const int c = threadIdx.x + blockDim.x * i;
            // slots in order j = 0..k-1, then the shared slices in order, then onto h
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < kCombineSlots + kCombineShared; ++j) {
                acc.x += q[i][j].x;
                acc.y += q[i][j].y;
                acc.z += q[i][j].z;
                acc.w += q[i][j].w;
            }
            float4 o = q[i][kCombineSlots + kCombineShared];
            o.x += acc.x;
            o.y += acc.y;
            o.z += acc.z;
            o.w += acc.w;
            v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c < d4) {
                hr[c] = o;
                v[i] = o;
            }
        }
    } else {
#pragma unroll 1
        for (int i = 0; i < kRowCols; ++i) {
            const int c = threadIdx.x + blockDim.x * i;
            v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c >= d4) continue;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int sp = 0; sp < y_splits; ++sp)
                for (int j = 0; j < k; ++j) {
                    const float4 a = __ldg(reinterpret_cast<const float4*>(y + sp * y_split_stride +
                                                                          static_cast<size_t>(s_r[j]) * d) + c);
                    acc.x += a.x;
                    acc.y += a.y;
                    acc.z += a.z;
                    acc.w += a.w;
                }
            for (int j = 0; j < n_shared; ++j) {
                const float4 a =
                    __ldg(reinterpret_cast<const float4*>(y_shared + (static_cast<size_t>(j) * rows + t) * d) + c);
                acc.x += a.x;
                acc.y += a.y;
                acc.z += a.z;
                acc.w += a.w;
            }
            float4 o = hr[c];
            o.x += acc.x;
            o.y += acc.y;
            o.z += acc.z;
            o.w += acc.w;
            hr[c] = o;
            v[i] = o;
        }
    }
    if (g) norm_row_store<kRowCols>(v, d4, g, y_norm + static_cast<size_t>(t) * d, eps, red);
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

// ------------------------------------------------------------------ E4M3 rows
// Quantizes bf16 rows to E4M3 with one power-of-two scale per row (one warp per
// row, the row held in registers: cols / 256 uint4 per lane, cols a multiple of
// 8, at most 4096).  Source column c goes to destination column
// (c / slice) * slice_pad + c % slice: slice = cols packs the row, slice < cols
// spreads it into zero-padded slices (the shared FFN's activation, whose
// feature slices are read as separate K ranges of 128-element blocks).
constexpr int kQuantMaxV = 16;  // uint4 per lane: rows up to 4096 bf16
__global__ void quant_rows_e4m3_kernel(const bf16* __restrict__ src, size_t src_ld, int rows, int cols,
                                       uint8_t* __restrict__ dst, size_t dst_ld, int slice, int slice_pad,
                                       float* __restrict__ scale) {
    pdl_enter();
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const uint4* s = reinterpret_cast<const uint4*>(src + static_cast<size_t>(row) * src_ld);
    const int c8 = cols / 8;
    uint4 v[kQuantMaxV];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < kQuantMaxV; ++i) {
        const int c = lane + 32 * i;
        v[i] = c < c8 ? __ldg(&s[c]) : make_uint4(0, 0, 0, 0);
        amax = fmaxf(amax, bf16x8_absmax(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float sc, inv;
    e4m3_row_scale(amax, sc, inv);
    uint8_t* d = dst + static_cast<size_t>(row) * dst_ld;
#pragma unroll
    for (int i = 0; i < kQuantMaxV; ++i) {
        const int c = lane + 32 * i;
        if (c < c8) {
            const int e = 8 * c;
            *reinterpret_cast<uint2*>(d + (e / slice) * slice_pad + e % slice) = bf16x8_to_e4m3(v[i], inv);
        }
    }
    if (lane == 0) scale[row] = sc;
}

__global__ void set_inv_tau_kernel(float* p, float inv_tau_log2) {
    pdl_enter();
    *p = inv_tau_log2;
}

// Per-(row, 256-column tile) statistics of given fp32 logits (same format as the
// LM head epilogue writes: max, S, argmax and, when pent is not null, T).  One
// warp per (row, tile).
__global__ void stats_from_logits_kernel(const float* __restrict__ logits, int rows, int V, const float* inv_tau,
                                         float* __restrict__ pmax, float* __restrict__ psum, int* __restrict__ parg,
                                         float* __restrict__ pent) {
    pdl_enter();
    const int n_tiles = V / 256;
    const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= rows * n_tiles) return;
    const int row = w / n_tiles, tile = w % n_tiles;
    const float k = __ldg(inv_tau);
    const float* src = logits + static_cast<size_t>(row) * V + tile * 256;
    RowStat st{-INFINITY, 0.f, 0};
    float x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int c = j * 32 + lane;
        x[j] = __ldg(&src[c]);
        const RowStat one{x[j], 1.f, tile * 256 + c};
        st = stat_merge(st, one, k);
    }
    st = warp_stat(st, k);
    if (lane == 0) {
        pmax[w] = st.m;
        psum[w] = st.s;
        parg[w] = st.a;
    }
    if (pent) {  // T = sum 2^y y, y = (L - max) k, against the tile's max
        float t = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float y = (x[j] - st.m) * k;
            t = fmaf(exp2f(y), y, t);
        }
        t = warp_sum(t);
        if (lane == 0) pent[w] = t;
    }
}

// Per row: merge the vocab-tile statistics -> confidence = -log(sum) (the log of
// the largest tempered probability) and the argmax.  One warp per row.
__global__ void stats_combine_kernel(const float* __restrict__ pmax, const float* __restrict__ psum,
                                     const int* __restrict__ parg, int rows, int n_tiles, const float* inv_tau,
                                     float* __restrict__ conf, int* __restrict__ argmax) {
    pdl_enter();
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

// ------------------------------------------------------------------ self-conditioning
// p0_hat = Softmax(L / tau) rounded to bf16 (hyper.ai digest, Method, eq. 4):
// p[r][v] = exp2((L[r][v] - M) k) / S, k = log2(e) / tau, with the row's M and S
// merged from the LM head's per-tile statistics.  `slices` blocks of 256 threads
// per row, each merging the row's tiles itself and writing V / slices columns
// (V / slices a multiple of 4).
__global__ void __launch_bounds__(256) sc_probs_kernel(const float* __restrict__ logits,
                                                       const float* __restrict__ pmax, const float* __restrict__ psum,
                                                       int n_tiles, int V, const float* __restrict__ inv_tau,
                                                       bf16* __restrict__ p, int slices) {
    pdl_enter();
    __shared__ RowStat part[8];
    const int row = blockIdx.x / slices, sl = blockIdx.x - row * slices;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const float k = __ldg(inv_tau);
    RowStat st{-INFINITY, 0.f, 0};
    for (int t = threadIdx.x; t < n_tiles; t += blockDim.x) {
        const size_t o = static_cast<size_t>(row) * n_tiles + t;
        st = stat_merge(st, RowStat{pmax[o], psum[o], 0}, k);
    }
    st = warp_stat(st, k);
    if (lane == 0) part[w] = st;
    __syncthreads();
    st = part[0];
    for (int i = 1; i < (blockDim.x >> 5); ++i) st = stat_merge(st, part[i], k);
    const float M = st.m, inv_s = 1.f / st.s;
    const int per4 = V / slices / 4;
    const float4* src = reinterpret_cast<const float4*>(logits + static_cast<size_t>(row) * V) + sl * per4;
    uint2* dst = reinterpret_cast<uint2*>(p + static_cast<size_t>(row) * V) + sl * per4;
#pragma unroll 4
    for (int i = threadIdx.x; i < per4; i += blockDim.x) {
        const float4 l = __ldcs(&src[i]);
        dst[i] = make_uint2(pack2_bf16(exp2f((l.x - M) * k) * inv_s, exp2f((l.y - M) * k) * inv_s),
                            pack2_bf16(exp2f((l.z - M) * k) * inv_s, exp2f((l.w - M) * k) * inv_s));
    }
}

// u = sum of the n_parts K-split partials of p0_hat E (split order), then the
// FFW's pre-norm y = RMSNorm(u) with gain (1 + g), bf16.  One 128-thread block per row.
__global__ void __launch_bounds__(128) sc_norm_kernel(const float* __restrict__ u, int n_parts, size_t part_stride,
                                                      int rows, int d, const uint16_t* __restrict__ g,
                                                      bf16* __restrict__ y, float eps) {
    pdl_enter();
    __shared__ float red[4];
    const int row = blockIdx.x;
    if (row >= rows) return;
    const int d4 = d / 4;
    float4 v[kRowMaxV];
#pragma unroll
    for (int i = 0; i < kRowMaxV; ++i) {
        const int c = threadIdx.x + 128 * i;
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c < d4) {
            const float4* src = reinterpret_cast<const float4*>(u + static_cast<size_t>(row) * d) + c;
            for (int s = 0; s < n_parts; ++s) {
                const float4 a = src[s * (part_stride / 4)];
                v[i].x += a.x;
                v[i].y += a.y;
                v[i].z += a.z;
                v[i].w += a.w;
            }
        }
    }
    norm_row_store<kRowMaxV>(v, d4, g, y + static_cast<size_t>(row) * d, eps, red);
}

// ------------------------------------------------------------------ sampler
// One CTA per canvas, one thread per position.  Rank of an open position =
// number of open positions with larger confidence, or equal confidence and a
// lower index.  The m best are committed to their argmax and frozen; the other
// open positions are redrawn from Philox(seed; (pos_off + i, s, b, 1)), lane 0
// (pos_off = block index x C for the blocks after the first of a sequence).
__global__ void __launch_bounds__(1024)
    sample_commit_kernel(int32_t* __restrict__ tok, uint8_t* __restrict__ committed, const float* __restrict__ conf,
                         const int* __restrict__ argmax, int C, uint32_t V, int s, int last_step, int m_commit,
                         uint32_t pos_off, uint32_t k0, uint32_t k1, float* __restrict__ conf_out) {
    pdl_enter();
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
            const Philox4 r = philox4x32_10(pos_off + static_cast<uint32_t>(i), static_cast<uint32_t>(s),
                                            static_cast<uint32_t>(b), TAG_RENOISE, k0, k1);
            tok[o] = uniform_token(r.x, V);
        }
    }
    if (in && conf_out) conf_out[o] = c;
}

__global__ void init_canvas_kernel(int32_t* __restrict__ tok, uint8_t* __restrict__ committed, int B, int C,
                                   uint32_t V, uint32_t pos_off, uint32_t k0, uint32_t k1) {
    pdl_enter();
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= B * C) return;
    const int b = idx / C, i = idx % C;
    const Philox4 r =
        philox4x32_10(pos_off + static_cast<uint32_t>(i), 0u, static_cast<uint32_t>(b), TAG_INIT, k0, k1);
    tok[idx] = uniform_token(r.x, V);
    committed[idx] = 0;
}

// x_t = x0 if lane 1 < threshold (= floor(kappa 2^32)), else the uniform token of lane 0
__global__ void forward_noise_kernel(const int32_t* __restrict__ x0, int32_t* __restrict__ xt, int B, int C,
                                     uint32_t V, int step, uint64_t threshold, uint32_t k0, uint32_t k1) {
    pdl_enter();
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= B * C) return;
    const int b = idx / C, i = idx % C;
    const Philox4 r = philox4x32_10(static_cast<uint32_t>(i), static_cast<uint32_t>(step), static_cast<uint32_t>(b),
                                    TAG_FORWARD, k0, k1);
    xt[idx] = (static_cast<uint64_t>(r.y) < threshold) ? x0[idx] : uniform_token(r.x, V);
}

}  // namespace dgen
