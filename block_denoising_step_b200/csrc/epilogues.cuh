// Epilogue functors of the tcgen05 GEMM core.
//
// run<BN>(sched, item, taddr, q, lane, smem) is called by each of the four
// epilogue warps once the item's accumulator is complete.  taddr addresses
// TMEM lane (32 q) of the accumulator, column 0; thread `lane` of the warp owns
// accumulator row 32 q + lane.  tcgen05.ld is warp-collective, so every thread
// executes the loads; only the stores are predicated.
//
// Normal orientation (A = activation rows, B = weight rows): accumulator row =
// token row, column = output feature.  Swap-AB (grouped experts): accumulator
// row = output feature, column = token of the chunk.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace dgen {

__device__ __forceinline__ float gelu_tanh(float x) {
    // 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))  (Hendrycks & Gimpel 2016, tanh form)
    const float k0 = 0.7978845608028654f, k1 = 0.044715f;
    return 0.5f * x * (1.0f + tanhf(k0 * (x + k1 * x * x * x)));
}

// ------------------------------------------------------------------ D fp32 store (diagnostic GEMM)
// With a K split, split ks writes its partial product at d + ks * split_stride.
struct EpiStoreF32 {
    float* d;
    int M, N, ldd;
    size_t split_stride = 0;
    template <int BN>
    __device__ __forceinline__ void run(const tc::DenseSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t*) const {
        const int row = sc.m_of(it) * tc::BM + q * 32 + lane;
        const int col0 = sc.n_of(it) * BN;
        float* base = d + static_cast<size_t>(sc.ks_of(it)) * split_stride;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            uint32_t r[32];
            tmem_ld32(taddr + c, r);
            tmem_ld_wait();
            if (row < M) {
                float* dst = base + static_cast<size_t>(row) * ldd + col0 + c;
                if (col0 + c + 32 <= N && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {  // 16-byte stores
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        reinterpret_cast<float4*>(dst)[j] =
                            make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                        __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (col0 + c + j < N) dst[j] = __uint_as_float(r[j]);
                }
            }
        }
    }
};

// ------------------------------------------------------------------ per-row tile sums (streaming measurement)
// Writes one float per (row, column tile): the sum of the row's BN outputs.
struct EpiRowSum {
    float* out;  // [M][n_tiles]
    int M, n_tiles;
    template <int BN>
    __device__ __forceinline__ void run(const tc::DenseSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t*) const {
        const int row = sc.m_of(it) * tc::BM + q * 32 + lane;
        float acc = 0.f;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            uint32_t r[32];
            tmem_ld32(taddr + c, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) acc += __uint_as_float(r[j]);
        }
        if (row < M) out[static_cast<size_t>(row) * n_tiles + sc.n_of(it)] = acc;
    }
};

// ------------------------------------------------------------------ QKV: RoPE and scatter to Q / KV cache
// The packed projection has (Hq + 2 Hkv) heads of hd features: q heads, then
// k heads, then v heads.  A tile of BN columns holds BN / hd whole heads.
// q and k are rotated (rotate-half pairs (j, j + hd/2), angle pos * base^(-2j/hd),
// cos/sin from a table) and rounded to bf16 once.
struct EpiQKV {
    bf16* q_out;          // [B][Hq][n_q][hd]
    bf16* k_cache;        // [B][Hkv][S_max][hd] of this layer
    bf16* v_cache;
    const float2* rope;   // [S_max][hd/2] (cos, sin)
    int rows, n_q, pos0, Hq, Hkv, hd, S_max;
    template <int BN>
    __device__ __forceinline__ void run(const tc::DenseSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t*) const {
        const int row = sc.m_of(it) * tc::BM + q * 32 + lane;
        const bool live = row < rows;
        const int b = live ? row / n_q : 0;
        const int i = live ? row - b * n_q : 0;
        const int pos = pos0 + i;
        const int half = hd >> 1;
#pragma unroll 1
        for (int hc = 0; hc < BN; hc += hd) {
            const int head = (sc.n_of(it) * BN + hc) / hd;
            bf16* dst;
            bool rotate = true;
            if (head < Hq) {
                dst = q_out + ((static_cast<size_t>(b) * Hq + head) * n_q + i) * hd;
            } else if (head < Hq + Hkv) {
                dst = k_cache + ((static_cast<size_t>(b) * Hkv + (head - Hq)) * S_max + pos) * hd;
            } else {
                dst = v_cache + ((static_cast<size_t>(b) * Hkv + (head - Hq - Hkv)) * S_max + pos) * hd;
                rotate = false;
            }
#pragma unroll 1
            for (int c = 0; c < half; c += 32) {
                uint32_t r1[32], r2[32];
                tmem_ld32(taddr + hc + c, r1);
                tmem_ld32(taddr + hc + half + c, r2);
                tmem_ld_wait();
                if (!live) continue;
                uint32_t o1[16], o2[16];
                const float2* cs = rope + static_cast<size_t>(pos) * half + c;
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    float a0 = __uint_as_float(r1[j]), a1 = __uint_as_float(r1[j + 1]);
                    float b0 = __uint_as_float(r2[j]), b1 = __uint_as_float(r2[j + 1]);
                    if (rotate) {
                        const float2 t0 = cs[j], t1 = cs[j + 1];
                        const float x0 = a0 * t0.x - b0 * t0.y, y0 = b0 * t0.x + a0 * t0.y;
                        const float x1 = a1 * t1.x - b1 * t1.y, y1 = b1 * t1.x + a1 * t1.y;
                        a0 = x0; b0 = y0; a1 = x1; b1 = y1;
                    }
                    o1[j >> 1] = pack2_bf16(a0, a1);
                    o2[j >> 1] = pack2_bf16(b0, b1);
                }
                uint4* d1 = reinterpret_cast<uint4*>(dst + c);
                uint4* d2 = reinterpret_cast<uint4*>(dst + half + c);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    d1[j] = make_uint4(o1[4 * j], o1[4 * j + 1], o1[4 * j + 2], o1[4 * j + 3]);
                    d2[j] = make_uint4(o2[4 * j], o2[4 * j + 1], o2[4 * j + 2], o2[4 * j + 3]);
                }
            }
        }
    }
};

// Same for hd > BN with PairSched tiles (BN = hd / 2): tile n holds features
// f0 + [0, BN/2) of head n / 2 in columns [0, BN/2) and their rotate-half
// partners f0 + hd/2 + [0, BN/2) in columns [BN/2, BN), f0 = (n % 2) * BN/2.
struct EpiQKVPair {
    bf16* q_out;          // [B][Hq][n_q][hd]
    bf16* k_cache;        // [B][Hkv][S_max][hd] of this layer
    bf16* v_cache;
    const float2* rope;   // [S_max][hd/2] (cos, sin)
    int rows, n_q, pos0, Hq, Hkv, hd, S_max;
    template <int BN>
    __device__ __forceinline__ void run(const tc::PairSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t*) const {
        constexpr int HB = BN / 2;
        const int row = sc.m_of(it) * tc::BM + q * 32 + lane;
        const bool live = row < rows;
        const int b = live ? row / n_q : 0;
        const int i = live ? row - b * n_q : 0;
        const int pos = pos0 + i;
        const int half = hd >> 1;
        const int per = hd / BN, n = sc.n_of(it);
        const int head = n / per, f0 = (n % per) * HB;
        bf16* dst;
        bool rotate = true;
        if (head < Hq) {
            dst = q_out + ((static_cast<size_t>(b) * Hq + head) * n_q + i) * hd;
        } else if (head < Hq + Hkv) {
            dst = k_cache + ((static_cast<size_t>(b) * Hkv + (head - Hq)) * S_max + pos) * hd;
        } else {
            dst = v_cache + ((static_cast<size_t>(b) * Hkv + (head - Hq - Hkv)) * S_max + pos) * hd;
            rotate = false;
        }
#pragma unroll 1
        for (int c = 0; c < HB; c += 32) {
            uint32_t r1[32], r2[32];
            tmem_ld32(taddr + c, r1);
            tmem_ld32(taddr + HB + c, r2);
            tmem_ld_wait();
            if (!live) continue;
            uint32_t o1[16], o2[16];
            const float2* cs = rope + static_cast<size_t>(pos) * half + f0 + c;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                float a0 = __uint_as_float(r1[j]), a1 = __uint_as_float(r1[j + 1]);
                float b0 = __uint_as_float(r2[j]), b1 = __uint_as_float(r2[j + 1]);
                if (rotate) {
                    const float2 t0 = cs[j], t1 = cs[j + 1];
                    const float x0 = a0 * t0.x - b0 * t0.y, y0 = b0 * t0.x + a0 * t0.y;
                    const float x1 = a1 * t1.x - b1 * t1.y, y1 = b1 * t1.x + a1 * t1.y;
                    a0 = x0; b0 = y0; a1 = x1; b1 = y1;
                }
                o1[j >> 1] = pack2_bf16(a0, a1);
                o2[j >> 1] = pack2_bf16(b0, b1);
            }
            uint4* d1 = reinterpret_cast<uint4*>(dst + f0 + c);
            uint4* d2 = reinterpret_cast<uint4*>(dst + half + f0 + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                d1[j] = make_uint4(o1[4 * j], o1[4 * j + 1], o1[4 * j + 2], o1[4 * j + 3]);
                d2[j] = make_uint4(o2[4 * j], o2[4 * j + 1], o2[4 * j + 2], o2[4 * j + 3]);
            }
        }
    }
};

// ------------------------------------------------------------------ experts: GELU(gate) * up -> bf16
// Swap-AB tile of the gate-up GEMM (GroupedSched over 16-row interleaved
// weights): in warp q, lanes 0..15 hold gate features mt*64 + 16q + lane and
// lanes 16..31 the matching up features; columns are the chunk's tokens.
// Shared-FFN chunks (expert id E + j) write features j*w + f of act_sh.
// E4M3 operands (w_scale set): the accumulator is first multiplied by the weight
// row's scale (stored row e*2w + mt*128 + TMEM lane; pseudo-expert j: row
// j*2w + ... of the shared tensor) and the token row's scale (the permuted row
// for routed chunks, the token row for shared ones).
struct EpiGateUp {
    bf16* act;      // [permuted rows][width]
    int width;      // w (row stride of act)
    int E = 0x7fffffff;
    bf16* act_sh = nullptr;  // [token rows][width_sh]
    int width_sh = 0;
    const float* w_scale = nullptr;     // [E][2w]   (E4M3 weights)
    const float* w_scale_sh = nullptr;  // [2 ws]
    const float* x_scale = nullptr;     // [permuted rows]
    const float* x_scale_sh = nullptr;  // [token rows]
    template <int BN>
    __device__ __forceinline__ void run(const tc::GroupedSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t*) const {
        const int4 ch = sc.chunk(it);
        int f = sc.mt_of(it) * 64 + q * 16 + (lane & 15);
        bf16* out = act;
        int stride = width;
        bool ok = true;
        const bool sh = ch.x >= E;
        if (sh) {
            f += (ch.x - E) * width;
            out = act_sh;
            stride = width_sh;
            ok = f < width_sh;
        }
        float wsc = 1.f;
        const float* xs = nullptr;
        if (w_scale) {
            const int wrow = (sh ? ch.x - E : ch.x) * 2 * width + sc.mt_of(it) * tc::BM + q * 32 + lane;
            wsc = sh ? (ok ? __ldg(&w_scale_sh[wrow]) : 0.f) : __ldg(&w_scale[wrow]);
            xs = sh ? x_scale_sh : x_scale;
        }
#pragma unroll 1
        for (int c = 0; c < BN && c < ch.z; c += 32) {  // only the chunk's columns
            uint32_t r[32];
            tmem_ld32(taddr + c, r);
            const float xl = (xs && c + lane < ch.z) ? __ldg(&xs[ch.y + c + lane]) : 1.f;
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float a = __uint_as_float(r[j]) * (wsc * __shfl_sync(0xffffffffu, xl, j));
                const float up = __shfl_down_sync(0xffffffffu, a, 16);
                if (lane < 16 && ok && c + j < ch.z) {
                    const float v = gelu_tanh(a) * up;
                    out[static_cast<size_t>(ch.y + c + j) * stride + f] = __float2bfloat16_rn(v);
                }
            }
        }
    }
};

// ------------------------------------------------------------------ dense gated GELU (self-conditioning FFW)
// Normal orientation: accumulator row = token row, columns = stored gate-up
// rows, interleaved in blocks of 16 (columns 32j..32j+15 gate features
// 16j..16j+15, columns 32j+16..32j+31 the matching up features), so each
// 32-column load gives 16 activations act[row][16 j + i] = GELU(gate) * up, bf16.
struct EpiGateUpDense {
    bf16* act;   // [rows][width]
    int width, rows;
    template <int BN>
    __device__ __forceinline__ void run(const tc::DenseSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t*) const {
        const int row = sc.m_of(it) * tc::BM + q * 32 + lane;
        const int col0 = sc.n_of(it) * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            uint32_t r[32];
            tmem_ld32(taddr + c, r);
            tmem_ld_wait();
            if (row < rows) {
                uint32_t o[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    o[j] = pack2_bf16(gelu_tanh(__uint_as_float(r[2 * j])) * __uint_as_float(r[16 + 2 * j]),
                                      gelu_tanh(__uint_as_float(r[2 * j + 1])) * __uint_as_float(r[17 + 2 * j]));
                uint4* dst = reinterpret_cast<uint4*>(act + static_cast<size_t>(row) * width + (col0 + c) / 2);
                dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
    }
};

// ------------------------------------------------------------------ experts: down projection * gate -> fp32 rows
// Shared-FFN chunks (expert id E + j) write part j of y_sh, gate 1.  E4M3
// operands (w_scale set): the accumulator is multiplied by the output row's
// weight scale and the activation row's scale before the gate.
struct EpiDown {
    float* y;            // [permuted rows][d] (+ ks * split_stride for K split ks)
    const float* gate;   // [permuted rows] or null (gate 1)
    int d;
    size_t split_stride = 0;
    int E = 0x7fffffff;
    float* y_sh = nullptr;  // [pseudo-experts][token rows][d]
    size_t sh_stride = 0;   // token rows * d
    const float* w_scale = nullptr;     // [E][d]  (E4M3 weights)
    const float* w_scale_sh = nullptr;  // [d]
    const float* a_scale = nullptr;     // [permuted rows]
    const float* a_scale_sh = nullptr;  // [token rows]
    template <int BN>
    __device__ __forceinline__ void run(const tc::GroupedSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t*) const {
        const int4 ch = sc.chunk(it);
        const int o = sc.mt_of(it) * tc::BM + q * 32 + lane;
        const bool sh = ch.x >= E;
        float* ybase = (sh ? y_sh + (ch.x - E) * sh_stride : y + sc.ks_of(it) * split_stride) +
                       static_cast<size_t>(ch.y) * d + o;
        const float* g_src = sh ? nullptr : gate;
        const float wsc = w_scale ? (sh ? __ldg(&w_scale_sh[o]) : __ldg(&w_scale[static_cast<size_t>(ch.x) * d + o]))
                                  : 1.f;
        const float* as = w_scale ? (sh ? a_scale_sh : a_scale) : nullptr;
#pragma unroll 1
        for (int c = 0; c < BN && c < ch.z; c += 32) {  // only the chunk's columns
            uint32_t r[32];
            tmem_ld32(taddr + c, r);
            // the chunk's gates (and activation scales) for these 32 columns, one load per lane
            float gl = (g_src && c + lane < ch.z) ? __ldg(&g_src[ch.y + c + lane]) : 1.0f;
            if (as && c + lane < ch.z) gl *= __ldg(&as[ch.y + c + lane]);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float g = __shfl_sync(0xffffffffu, gl, j);
                if (c + j < ch.z) ybase[static_cast<size_t>(c + j) * d] = (__uint_as_float(r[j]) * wsc) * g;
            }
        }
    }
};

// ------------------------------------------------------------------ both expert GEMMs in one launch
// Gate-up items run EpiGateUp and then signal their chunk: each lane fences its
// activation stores for the async proxy (the down items read them by TMA), the
// warp synchronises, and lane 0 releases one count on ready[chunk] (four warps
// per item).  Down items run EpiDown.
struct EpiFusedExpert {
    EpiGateUp gu;
    EpiDown dn;
    int* ready;
    template <int BN>
    __device__ __forceinline__ void run(const tc::FusedExpertSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t* sm) const {
        const int g = sc.n_gu();
        if (it < g) {
            gu.template run<BN>(sc.gu, it, taddr, q, lane, sm);
            fence_proxy_async_global();
            __syncwarp();
            if (lane == 0) {
                __threadfence();
                atomicAdd(&ready[it / sc.gu.m_tiles], 1);
            }
        } else {
            dn.template run<BN>(sc.dn, it - g, taddr, q, lane, sm);
        }
    }
};

// ------------------------------------------------------------------ LM head: per-(row, vocab tile) softmax statistics
// For row r and vocab tile n (BN columns), with y_j = (L_j - max) / tau in log2
// units (y_j = (L_j - max) k, k = log2(e) / tau): the max logit, its first column
// (global vocab index), S = sum_j 2^y_j and T = sum_j 2^y_j y_j, accumulated
// online over 32-column chunks (when the max grows by dy < 0 in log2 units the
// old terms scale by f = 2^dy and shift by dy: S' = f S, T' = f (T + S dy)).
// S gives the confidence of the tempered softmax, T / S its entropy
// (H = ln S - ln 2 T / S nats).  Optionally stores the fp32 logits.
struct EpiLMHead {
    float* pmax;          // [rows][n_tiles]
    float* psum;
    float* pent;          // [rows][n_tiles]: T
    int* parg;
    float* logits;        // [rows][V] or null
    const float* inv_tau; // device scalar: log2(e) / tau
    int rows, V, n_tiles;
    template <int BN>
    __device__ __forceinline__ void run(const tc::DenseSched& sc, int it, uint32_t taddr, int q, int lane,
                                        uint8_t*) const {
        const int row = sc.m_of(it) * tc::BM + q * 32 + lane;
        const int n = sc.n_of(it);
        const int col0 = n * BN;
        const float k = __ldg(inv_tau);
        float M = -INFINITY, S = 0.f, T = 0.f;
        int A = 0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            uint32_t r[32];
            tmem_ld32(taddr + c, r);
            tmem_ld_wait();
            float cm = __uint_as_float(r[0]);
            int ca = 0;
#pragma unroll
            for (int j = 1; j < 32; ++j) {
                const float v = __uint_as_float(r[j]);
                if (v > cm) {
                    cm = v;
                    ca = j;
                }
            }
            if (cm > M) {
                if (M == -INFINITY) {
                    S = 0.f;
                    T = 0.f;
                } else {
                    const float dy = (M - cm) * k;
                    const float f = exp2f(dy);
                    T = f * fmaf(S, dy, T);
                    S *= f;
                }
                M = cm;
                A = col0 + c + ca;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float y = (__uint_as_float(r[j]) - M) * k;
                const float e = exp2f(y);
                S += e;
                T = fmaf(e, y, T);
            }
            if (logits && row < rows) {
                float4* dst = reinterpret_cast<float4*>(logits + static_cast<size_t>(row) * V + col0 + c);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    __stcs(dst + j, make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                                __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
            }
        }
        if (row < rows) {
            const size_t o = static_cast<size_t>(row) * n_tiles + n;
            pmax[o] = M;
            psum[o] = S;
            pent[o] = T;
            parg[o] = A;
        }
    }
};

}  // namespace dgen
