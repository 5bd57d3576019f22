// Attention of a block of query rows over a key range of the KV cache, with an
// online (running max / running sum) softmax, split over key chunks.
//
//   o_i = sum_j softmax_j(q_i . k_j / sqrt(hd)) v_j
//
// Canvas pass: queries are the canvas rows at positions P..P+C-1 and the keys
// are ALL of [prompt cache ; canvas] with no mask (the decoder's bidirectional
// attention plus attention to the cache; hyper.ai digest of the DiffusionGemma
// paper, Method, three-stage pipeline).  Prompt pass: queries are the prompt
// rows and key j is visible to query i only if j <= i (causal encoder).
//
// One CTA = 4 warps x 16 query rows of one (sequence, query head, key split).
// Q.K^T and P.V run on mma.sync m16n8k16 bf16 -> fp32; K/V tiles of 64 keys
// are double-buffered in shared memory (16-byte chunks XOR-swizzled by row)
// with cp.async.  GQA: query head h reads KV head h * Hkv / Hq.
#pragma once

#include "common.cuh"

namespace dgen {

constexpr int kMaxAttnSplits = 32;  // key splits of one attention launch (one warp lane each)

struct AttnArgs {
    const bf16* q;     // [B][Hq][n_q][hd]
    const bf16* k;     // [B][Hkv][S_max][hd]
    const bf16* v;
    bf16* o;           // [B * n_q][Hq * hd]   (used when n_splits == 1)
    float* part_o;     // [n_splits][B][Hq][n_q][hd] (normalised per split)
    float* part_lse;   // [n_splits][B][Hq][n_q]     (log2 domain)
    int B, Hq, Hkv, n_q, S, S_max;
    int q_pos0;        // absolute position of query row 0 (causal pass)
    int causal;
    int n_splits, keys_per_split;
    float scale_log2;  // log2(e) / sqrt(hd)
};

namespace attn {

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    const int sz = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (a, b) -> bf16x2 hi = RNE(a, b) and lo = RNE((a, b) - hi)
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack2_bf16(a, b);
    const float2 h = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
    lo = pack2_bf16(a - h.x, b - h.y);
}

// byte offset of element (r, c) (c a multiple of 8) in a [rows][HD] bf16 tile
template <int HD>
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return static_cast<uint32_t>((r * HD + ((((c >> 3) ^ (r & 7))) << 3)) * 2);
}

template <int HD>
__device__ __forceinline__ void load_tile(uint32_t sdst, const bf16* gsrc, int row0, int n_valid, int tid) {
    constexpr int CH = HD / 8;  // 16-byte chunks per row
#pragma unroll
    for (int id = tid; id < 64 * CH; id += 128) {
        const int r = id / CH, cc = id % CH;
        const bool valid = r < n_valid;
        const bf16* src = gsrc + static_cast<size_t>(valid ? row0 + r : row0) * HD + cc * 8;
        cp_async16(sdst + swz<HD>(r, cc * 8), src, valid);
    }
}

}  // namespace attn

template <int HD>
__global__ void __launch_bounds__(128) attention_kernel(const AttnArgs a) {
    pdl_enter();
    using namespace attn;
    constexpr int TILE = 64 * HD * 2;
    constexpr int NT_O = HD / 8;  // 8-wide output column tiles
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sQ = smem_u32(smem);
    const uint32_t sK0 = sQ + TILE, sV0 = sQ + 3 * TILE;  // K[2], V[2]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int qt = blockIdx.x, h = blockIdx.y;
    const int b = blockIdx.z / a.n_splits, split = blockIdx.z % a.n_splits;
    const int kvh = (h * a.Hkv) / a.Hq;
    const int i0 = qt * 64;

    int k_begin = split * a.keys_per_split;
    int k_end = min(a.S, k_begin + a.keys_per_split);
    if (a.causal) k_end = min(k_end, a.q_pos0 + min(i0 + 64, a.n_q));
    const int n_tiles = k_end > k_begin ? (k_end - k_begin + 63) / 64 : 0;

    const bf16* qg = a.q + ((static_cast<size_t>(b) * a.Hq + h) * a.n_q) * HD;
    const bf16* kg = a.k + ((static_cast<size_t>(b) * a.Hkv + kvh) * a.S_max) * HD;
    const bf16* vg = a.v + ((static_cast<size_t>(b) * a.Hkv + kvh) * a.S_max) * HD;

    load_tile<HD>(sQ, qg, i0, min(64, a.n_q - i0), tid);
    if (n_tiles > 0) {
        load_tile<HD>(sK0, kg, k_begin, min(64, k_end - k_begin), tid);
        load_tile<HD>(sV0, vg, k_begin, min(64, k_end - k_begin), tid);
    }
    cp_commit();

    float o[NT_O][4];
#pragma unroll
    for (int n = 0; n < NT_O; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    const int r_lo = warp * 16 + g;  // this thread's rows in the tile: r_lo, r_lo + 8
    const int qpos_lo = a.q_pos0 + i0 + r_lo, qpos_hi = qpos_lo + 8;

    for (int kt = 0; kt < n_tiles; ++kt) {
        const int buf = kt & 1;
        const int key0 = k_begin + kt * 64;
        if (kt + 1 < n_tiles) {
            const int nk = key0 + 64;
            load_tile<HD>(sK0 + (buf ^ 1) * TILE, kg, nk, min(64, k_end - nk), tid);
            load_tile<HD>(sV0 + (buf ^ 1) * TILE, vg, nk, min(64, k_end - nk), tid);
            cp_commit();
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncthreads();
        const uint32_t sK = sK0 + buf * TILE, sV = sV0 + buf * TILE;

        // S = Q K^T for this warp's 16 rows x 64 keys
        float s[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
            uint32_t qa0, qa1, qa2, qa3;
            ldsm_x4(sQ + swz<HD>(warp * 16 + (lane & 15), ks * 16 + (lane >> 4) * 8), qa0, qa1, qa2, qa3);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t k0, k1, k2, k3;
                ldsm_x4(sK + swz<HD>(np * 16 + (lane & 7) + ((lane >> 4) << 3), ks * 16 + ((lane >> 3) & 1) * 8),
                        k0, k1, k2, k3);
                mma16816(s[2 * np], qa0, qa1, qa2, qa3, k0, k1);
                mma16816(s[2 * np + 1], qa0, qa1, qa2, qa3, k2, k3);
            }
        }
        // scale, mask, running max
        float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < 8; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = key0 + n * 8 + 2 * t + (e & 1);
                const int qp = (e < 2) ? qpos_lo : qpos_hi;
                const bool ok = key < k_end && (!a.causal || key <= qp);
                const float v = ok ? s[n][e] * a.scale_log2 : -INFINITY;
                s[n][e] = v;
                mt[e >> 1] = fmaxf(mt[e >> 1], v);
            }
        }
        float corr[2], mu[2];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            mt[hr] = fmaxf(mt[hr], __shfl_xor_sync(0xffffffffu, mt[hr], 1));
            mt[hr] = fmaxf(mt[hr], __shfl_xor_sync(0xffffffffu, mt[hr], 2));
            const float m_new = fmaxf(m_run[hr], mt[hr]);
            mu[hr] = (m_new == -INFINITY) ? 0.f : m_new;
            corr[hr] = exp2f(m_run[hr] - mu[hr]);
            m_run[hr] = m_new;
            l_run[hr] *= corr[hr];
        }
#pragma unroll
        for (int n = 0; n < NT_O; ++n) {
            o[n][0] *= corr[0];
            o[n][1] *= corr[0];
            o[n][2] *= corr[1];
            o[n][3] *= corr[1];
        }
#pragma unroll
        for (int n = 0; n < 8; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p = exp2f(s[n][e] - mu[e >> 1]);
                s[n][e] = p;
                l_run[e >> 1] += p;
            }
        }
        // O += P V with P = P_hi + P_lo, both bf16 (P_lo = bf16(P - P_hi)): the
        // product keeps ~16 significant bits of P instead of bf16's 8, so the
        // attention output is exact to fp32 accumulation order.
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t ph[4], pl[4];
            split_bf16(s[2 * kk][0], s[2 * kk][1], ph[0], pl[0]);
            split_bf16(s[2 * kk][2], s[2 * kk][3], ph[1], pl[1]);
            split_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1], ph[2], pl[2]);
            split_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3], ph[3], pl[3]);
#pragma unroll
            for (int np = 0; np < HD / 16; ++np) {
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(sV + swz<HD>(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, np * 16 + (lane >> 4) * 8), v0,
                          v1, v2, v3);
                mma16816(o[2 * np], ph[0], ph[1], ph[2], ph[3], v0, v1);
                mma16816(o[2 * np + 1], ph[0], ph[1], ph[2], ph[3], v2, v3);
                mma16816(o[2 * np], pl[0], pl[1], pl[2], pl[3], v0, v1);
                mma16816(o[2 * np + 1], pl[0], pl[1], pl[2], pl[3], v2, v3);
            }
        }
        __syncthreads();
    }

    // finish: full row sums across the quad, normalise, store
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        l_run[hr] += __shfl_xor_sync(0xffffffffu, l_run[hr], 1);
        l_run[hr] += __shfl_xor_sync(0xffffffffu, l_run[hr], 2);
    }
    const float inv[2] = {l_run[0] > 0.f ? 1.f / l_run[0] : 0.f, l_run[1] > 0.f ? 1.f / l_run[1] : 0.f};
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int i = i0 + r_lo + hr * 8;
        if (i >= a.n_q) continue;
        if (a.n_splits == 1) {
            bf16* dst = a.o + (static_cast<size_t>(b) * a.n_q + i) * (a.Hq * HD) + h * HD;
#pragma unroll
            for (int n = 0; n < NT_O; ++n)
                *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * t) =
                    pack2_bf16(o[n][2 * hr] * inv[hr], o[n][2 * hr + 1] * inv[hr]);
        } else {
            const size_t rowi = ((static_cast<size_t>(split) * a.B + b) * a.Hq + h) * a.n_q + i;
            float* dst = a.part_o + rowi * HD;
#pragma unroll
            for (int n = 0; n < NT_O; ++n)
                *reinterpret_cast<float2*>(dst + n * 8 + 2 * t) =
                    make_float2(o[n][2 * hr] * inv[hr], o[n][2 * hr + 1] * inv[hr]);
            if (t == 0) a.part_lse[rowi] = l_run[hr] > 0.f ? m_run[hr] + log2f(l_run[hr]) : -INFINITY;
        }
    }
}

// o[b*n_q + i][h*hd + c] = sum_s w_s o_s / sum_s w_s,  w_s = 2^(lse_s - max lse)
// One warp per query row (8 rows per 256-thread block): lane s holds split s's
// log-sum-exp, each lane owns hd/32 consecutive columns; every split's columns
// are loaded before they are summed (in split order).
template <int HD>
__global__ void __launch_bounds__(256) attention_combine_kernel(const AttnArgs a) {
    pdl_enter();
    constexpr int CPL = HD / 32;  // columns per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;  // over B * Hq * n_q, ordered (b, h, i)
    const int rows = a.B * a.Hq * a.n_q;
    if (row >= rows) return;
    const int i = row % a.n_q, bh = row / a.n_q;
    const int h = bh % a.Hq, b = bh / a.Hq;
    const size_t stride = static_cast<size_t>(rows);
    const float my_lse = lane < a.n_splits ? __ldg(&a.part_lse[lane * stride + row]) : -INFINITY;
    float mx = my_lse;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float my_w = (my_lse == -INFINITY) ? 0.f : exp2f(my_lse - mx);
    float acc[CPL], wsum = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
#pragma unroll 4
    for (int s = 0; s < a.n_splits; ++s) {
        const float w = __shfl_sync(0xffffffffu, my_w, s);
        const float* src = a.part_o + (s * stride + row) * HD + lane * CPL;
        float v[CPL];
#pragma unroll
        for (int c = 0; c < CPL; c += 2) {
            const float2 t = __ldg(reinterpret_cast<const float2*>(src + c));
            v[c] = t.x;
            v[c + 1] = t.y;
        }
        wsum += w;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c] += w * v[c];
    }
    const float inv = 1.f / wsum;
    bf16* dst = a.o + (static_cast<size_t>(b) * a.n_q + i) * (a.Hq * HD) + h * HD + lane * CPL;
#pragma unroll
    for (int c = 0; c < CPL; c += 2)
        *reinterpret_cast<uint32_t*>(dst + c) = pack2_bf16(acc[c] * inv, acc[c + 1] * inv);
}

}  // namespace dgen
