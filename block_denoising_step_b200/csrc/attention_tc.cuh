// Canvas-pass attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
//   o_i = sum_j softmax_j(q_i . k_j / sqrt(hd)) v_j,  keys j = all of [prompt cache ; canvas]
//
// (the decoder's bidirectional attention over the canvas plus attention to the
// prompt's cache; hyper.ai digest of the DiffusionGemma paper, Method,
// three-stage pipeline).  No mask: every canvas query sees every key.  With
// a.causal set (the encoder's prompt pass and the causal append of a finished
// canvas) query i at position q_pos0 + i sees the keys at positions <= its own:
// each CTA stops at its last query's position and masks per row, and the CTAs
// are taken heaviest query tile first.
//
// One CTA = 128 query rows of one (sequence, query head) over one key split,
// 192 threads:
//   warp 0 lane 0   TMA producer: the Q tile once, then 64-key K and V tiles
//                   into a shared-memory ring in the order the MMAs use them
//                   (K0, K1, K2, V0, K3, V1, K4, ...);
//   warp 1 lane 0   MMA issuer: S_j = Q K_j^T into one of three TMEM buffers
//                   (128 x 64 fp32), and O += P_j V_j into the TMEM output
//                   accumulator (128 x hd fp32), with V read MN-major from
//                   shared memory and P_j read from TMEM (the A operand of a
//                   tensor-memory-sourced MMA: P_j lives in S_j's columns);
//   warps 2..5      softmax: thread = query row.  Each reads its S_j row from
//                   TMEM, keeps a running max m and sum l (exp2 domain), writes
//                   P_j = 2^(s - m) back over S_j as bf16 hi + lo parts (hi =
//                   bf16(P), lo = bf16(P - hi), so P.V keeps about 16
//                   significant bits of P; columns 0..31 hi, 32..63 lo, two keys
//                   per column) and, at the end, reads O back and stores O / l.
// The MMAs are issued S0, S1, S2, P0V0, S3, P1V1, S4, ...: while the softmax
// works on S_j the tensor cores have S_{j+1}, P_{j-2}V_{j-2}, P_{j-1}V_{j-1} and
// S_{j+2} queued, and S_{j+3} reuses S_j's buffer only after P_j V_j in issue
// order.  With no P in shared memory the K/V ring holds 5 tiles at hd = 256.
// The softmax waits for an earlier P.V only to rescale O.
// The running max is moved only when it grows by more than 2^8 (P entries stay
// below 256), and then O is rescaled in TMEM; the result is the same softmax.
// Partial results of a key split are stored normalised with their log2-sum-exp
// for attention_combine_kernel (the format of attention_kernel's splits).
// Every wait is bounded; on a timeout the kernel records an error, drains its
// own copies and MMAs, frees its tensor memory and exits.
#pragma once

#include "attention.cuh"
#include "common.cuh"

namespace dgen {
namespace attn_tc {

constexpr int BQ = 128;    // query rows per CTA (TMEM lanes)
constexpr int kThreads = 192;  // producer warp, MMA warp, 4 softmax warps
constexpr int BKEY = 64;   // keys per tile
constexpr int NB = 3;      // S / P buffers in TMEM
constexpr float kRescaleLog2 = 8.f;

template <int HD>
struct Layout {
    static constexpr int QB = HD / 64;                  // 64-column boxes per row
    static constexpr int Q_BYTES = BQ * HD * 2;         // QB boxes of [128 rows x 128 B]
    static constexpr int KV_BYTES = BKEY * HD * 2;      // QB boxes of [64 rows x 128 B]
    static constexpr int STAGES = HD == 256 ? 5 : 8;
    static constexpr int KV_OFF = Q_BYTES;
    static constexpr int BAR_OFF = KV_OFF + STAGES * KV_BYTES;
    // q_full, kv_full[STAGES], kv_empty[STAGES], s_full[NB], p_full[NB], pv_done[NB], drain
    static constexpr int N_BARS = 1 + 2 * STAGES + 3 * NB + 1;
    static constexpr int SLOT_OFF = BAR_OFF + N_BARS * 8;
    static constexpr int SMEM_BYTES = SLOT_OFF + 16 + 1024;  // + slack for 1024-byte alignment
    static constexpr int TMEM_COLS = (HD + NB * BKEY) <= 256 ? 256 : 512;  // O, then S/P[NB]
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(HD + NB * BKEY <= 512, "tensor memory");
};

// ring position -> (tile, K or V): K0..K_{NB-1}, then V_j followed by K_{j+NB},
// then the last V tiles (the order the MMA warp consumes them)
__device__ __forceinline__ void ring_item(int i, int n, int& tile, bool& is_k) {
    const int first = min(n, NB);
    if (i < first) {
        tile = i;
        is_k = true;
        return;
    }
    const int r = i - first, pairs = max(n - NB, 0);
    if (r < 2 * pairs) {
        is_k = (r & 1) != 0;
        tile = (r >> 1) + (is_k ? NB : 0);
    } else {
        is_k = false;
        tile = pairs + (r - 2 * pairs);
    }
}

// D (TMEM) (+)= A (TMEM, K-major: lane = row, two bf16 per 32-bit column) x
// B (shared-memory descriptor), kind::f16.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

}  // namespace attn_tc

template <int HD>
__global__ void __launch_bounds__(attn_tc::kThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnArgs a, int* __restrict__ err) {
    using namespace attn_tc;
    using L = Layout<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase, sKV = sbase + L::KV_OFF;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;
    uint64_t* kv_empty = kv_full + L::STAGES;
    uint64_t* s_full = kv_empty + L::STAGES;
    uint64_t* p_full = s_full + NB;
    uint64_t* pv_done = p_full + NB;
    uint64_t* drain = pv_done + NB;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SLOT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    int qt = blockIdx.x, h = blockIdx.y, bz = blockIdx.z;
    if (a.causal) {  // linear CTA order, query tiles with the most keys first
        const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
        const int per = gridDim.y * gridDim.z;
        qt = gridDim.x - 1 - lin / per;
        h = (lin % per) % gridDim.y;
        bz = (lin % per) / gridDim.y;
    }
    const int b = bz / a.n_splits, split = bz % a.n_splits;
    const int kvh = (h * a.Hkv) / a.Hq;
    const int k_begin = split * a.keys_per_split;
    int k_end = min(a.S, k_begin + a.keys_per_split);
    if (a.causal) k_end = min(k_end, a.q_pos0 + qt * BQ + BQ);  // the tile's last query position + 1
    const int n = k_end > k_begin ? (k_end - k_begin + BKEY - 1) / BKEY : 0;
    const int q_row0 = (b * a.Hq + h) * a.n_q + qt * BQ;
    const int kv_row0 = (b * a.Hkv + kvh) * a.S_max + k_begin;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int i = 0; i < NB; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_enter();  // Q and the canvas K / V come from the previous kernel
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_o = tmem, t_s = tmem + HD;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            if (n > 0) {
                mbar_expect_tx(q_full, L::Q_BYTES);
#pragma unroll
                for (int c = 0; c < L::QB; ++c)
                    tma_load_2d(sQ + c * (BQ * 128), &tmQ, c * 64, q_row0, smem_u32(q_full));
            }
            int s = 0;
            uint32_t ph = 0, pending = 0, fill_ph = 0;
            bool ok = true;
            for (int i = 0; i < 2 * n; ++i) {
                int tile;
                bool is_k;
                ring_item(i, n, tile, is_k);
                if (!mbar_wait(&kv_empty[s], ph ^ 1u, err, ERR_ATTN_PRODUCER)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_u32(&kv_full[s]);
                mbar_expect_tx(&kv_full[s], L::KV_BYTES);
                const uint32_t dst = sKV + s * L::KV_BYTES;
#pragma unroll
                for (int c = 0; c < L::QB; ++c)
                    tma_load_2d(dst + c * (BKEY * 128), is_k ? &tmK : &tmV, c * 64, kv_row0 + tile * BKEY, fb);
                pending |= 1u << s;
                fill_ph = (fill_ph & ~(1u << s)) | (ph << s);
                if (++s == L::STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (!ok) {  // let our own copies land before the CTA goes away
                if (n > 0) mbar_wait(q_full, 0, err, ERR_ATTN_DRAIN);
                for (int j = 0; j < L::STAGES; ++j)
                    if ((pending >> j) & 1u) mbar_wait(&kv_full[j], (fill_ph >> j) & 1u, err, ERR_ATTN_DRAIN);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(BQ, BKEY);
            constexpr uint32_t idesc_pv = idesc_bf16_f32_bmn(BQ, HD);
            int s = 0;
            uint32_t ph = 0;
            bool ok = n == 0 || mbar_wait(q_full, 0, err, ERR_ATTN_MMA);
            auto next_stage = [&](uint32_t& stage) -> bool {
                if (!mbar_wait(&kv_full[s], ph, err, ERR_ATTN_MMA)) return false;
                tc_fence_after();
                stage = s;
                if (++s == L::STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
                return true;
            };
            auto issue_s = [&](int j) -> bool {  // S_j = Q K_j^T
                uint32_t st;
                if (!next_stage(st)) return false;
                const uint32_t sk = sKV + st * L::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * (BQ * 128)) + 2 * (kk & 3);
                    const uint64_t bd = sdesc_sw128(sk + (kk >> 2) * (BKEY * 128)) + 2 * (kk & 3);
                    mma_bf16_ss(t_s + (j % NB) * BKEY, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(&kv_empty[st]));
                mma_commit(smem_u32(&s_full[j % NB]));
                return true;
            };
            for (int j = 0; ok && j < NB && j < n; ++j) ok = issue_s(j);
            for (int j = 0; ok && j < n; ++j) {
                if (!mbar_wait(&p_full[j % NB], (j / NB) & 1, err, ERR_ATTN_MMA)) break;
                tc_fence_after();
                uint32_t st;
                if (!next_stage(st)) break;
                const uint32_t sv = sKV + st * L::KV_BYTES;
                // O += P_hi V_j + P_lo V_j; P_j from TMEM (8 columns = 16 keys per MMA
                // step, hi in columns 0..31 of the buffer, lo in 32..63); V_j is
                // [64 keys][hd]: MN-major B, 64-column boxes BKEY * 128 bytes apart,
                // 16 keys = 2048 bytes per MMA step
                const uint32_t tp = t_s + (j % NB) * BKEY;
#pragma unroll
                for (int kk = 0; kk < BKEY / 16; ++kk) {
                    const uint64_t vd = sdesc_sw128_mn(sv + kk * 2048, BKEY * 128);
                    mma_bf16_ts(t_o, tp + kk * 8, vd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                    mma_bf16_ts(t_o, tp + BKEY / 2 + kk * 8, vd, idesc_pv, 1u);
                }
                mma_commit(smem_u32(&kv_empty[st]));
                mma_commit(smem_u32(&pv_done[j % NB]));
                if (j + NB < n && !issue_s(j + NB)) break;
            }
            mma_commit(smem_u32(drain));  // arrives when every MMA issued above has completed
            mbar_wait(drain, 0, err, ERR_ATTN_DRAIN);
        }
    } else {
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;
        // keys below lim are visible to this row (its own position included when causal)
        const int lim = a.causal ? min(k_end, a.q_pos0 + qt * BQ + row + 1) : k_end;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const uint32_t tb = t_s + (j % NB) * BKEY + lane_off;  // this warp's rows of buffer j % NB
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[j % NB], (j / NB) & 1, err, ERR_ATTN_SOFTMAX))) {
                ok = false;
                break;
            }
            tc_fence_after();
            float x[BKEY];  // raw scores q.k (masked keys -inf)
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(tb, r0);
                tmem_ld32(tb + 32, r1);
                tmem_ld_wait();
                const int key0 = k_begin + j * BKEY;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    x[c] = key0 + c < lim ? __uint_as_float(r0[c]) : -INFINITY;
                    x[32 + c] = key0 + 32 + c < lim ? __uint_as_float(r1[c]) : -INFINITY;
                }
            }
            // tile max (a tree, so the chain is 6 deep), in the exp2 domain (scale > 0)
            float mx[BKEY / 2];
#pragma unroll
            for (int c = 0; c < BKEY / 2; ++c) mx[c] = fmaxf(x[c], x[c + BKEY / 2]);
#pragma unroll
            for (int w = BKEY / 4; w >= 1; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; ++c) mx[c] = fmaxf(mx[c], mx[c + w]);
            const float mt = mx[0] * a.scale_log2;
            const bool move = mt > m_run + kRescaleLog2 || (m_run == -INFINITY && mt > -INFINITY);
            float corr = 1.f;
            if (move) {
                corr = m_run == -INFINITY ? 0.f : exp2f(m_run - mt);
                l_run *= corr;
                m_run = mt;
            }
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            // P = 2^(x scale - mu) as bf16 hi + lo pairs (two keys per 32-bit column):
            // hi = bf16(P), lo = bf16(P - hi), both rounded to nearest
            uint32_t hi[BKEY / 2], lo[BKEY / 2];
            float ps[BKEY / 2];
#pragma unroll
            for (int e = 0; e < BKEY / 2; ++e) {
                const float p0 = exp2f(fmaf(x[2 * e], a.scale_log2, -mu));
                const float p1 = exp2f(fmaf(x[2 * e + 1], a.scale_log2, -mu));
                ps[e] = p0 + p1;
                attn::split_bf16(p0, p1, hi[e], lo[e]);
            }
#pragma unroll
            for (int w = BKEY / 4; w >= 1; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; ++c) ps[c] += ps[c + w];
            l_run += ps[0];
            if (__any_sync(0xffffffffu, move && corr != 1.f && j > 0)) {  // rescale O rows in TMEM
                // after P_{j-1} V_{j-1} (and every earlier MMA) has completed, before P_j V_j
                if (!__all_sync(0xffffffffu,
                                mbar_wait(&pv_done[(j - 1) % NB], ((j - 1) / NB) & 1, err, ERR_ATTN_SOFTMAX))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < HD; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(t_o + c + lane_off, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * corr);
                    tmem_st32(t_o + c + lane_off, r);
                }
                tmem_st_wait();
            }
            // P_j over S_j (already read): hi in columns 0..31, lo in 32..63
            tmem_st32(tb, hi);
            tmem_st32(tb + BKEY / 2, lo);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[j % NB]);
        }
        if (ok && n > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(&pv_done[(n - 1) % NB], ((n - 1) / NB) & 1, err, ERR_ATTN_SOFTMAX)))
            ok = false;
        tc_fence_after();
        const int i = qt * BQ + row;
        const bool live = ok && i < a.n_q;
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        if (ok) {
            const size_t rowi = ((static_cast<size_t>(split) * a.B + b) * a.Hq + h) * a.n_q + i;
            // two 32-column loads in flight per wait (64 columns per round trip)
#pragma unroll 1
            for (int c0 = 0; c0 < HD; c0 += 64) {
                uint32_t rr[2][32];
                if (n > 0) {
                    tmem_ld32(t_o + c0 + lane_off, rr[0]);
                    tmem_ld32(t_o + c0 + 32 + lane_off, rr[1]);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) rr[0][e] = rr[1][e] = 0u;
                }
                if (!live) continue;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t(&r)[32] = rr[hh];
                    const int c = c0 + 32 * hh;
                    if (a.n_splits == 1) {
                        uint4* dst = reinterpret_cast<uint4*>(a.o + (static_cast<size_t>(b) * a.n_q + i) * (a.Hq * HD) +
                                                              h * HD + c);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(pack2_bf16(__uint_as_float(r[8 * e]) * inv, __uint_as_float(r[8 * e + 1]) * inv),
                                                pack2_bf16(__uint_as_float(r[8 * e + 2]) * inv, __uint_as_float(r[8 * e + 3]) * inv),
                                                pack2_bf16(__uint_as_float(r[8 * e + 4]) * inv, __uint_as_float(r[8 * e + 5]) * inv),
                                                pack2_bf16(__uint_as_float(r[8 * e + 6]) * inv, __uint_as_float(r[8 * e + 7]) * inv));
                    } else {
                        float4* dst = reinterpret_cast<float4*>(a.part_o + rowi * HD + c);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                                                 __uint_as_float(r[4 * e + 2]) * inv, __uint_as_float(r[4 * e + 3]) * inv);
                    }
                }
            }
            if (live && a.n_splits > 1) a.part_lse[rowi] = l_run > 0.f ? m_run + log2f(l_run) : -INFINITY;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace dgen
