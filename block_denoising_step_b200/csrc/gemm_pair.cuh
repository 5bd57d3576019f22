// The tcgen05 GEMM core on CTA pairs (cta_group::2).
//
// A pair of CTAs (a cluster of two, on two SMs) computes one 256 x BN output
// tile with tcgen05.mma.cta_group::2: CTA r holds rows 128 r .. 128 r + 127 of
// the A tile and rows r BN/2 .. r BN/2 + BN/2 - 1 of the B tile in its own
// shared memory, at the same offsets in both CTAs, and receives its 128 output
// rows x BN columns in its own tensor memory.  Each SM thus takes in 128 + BN/2
// rows per k-block for 128 x BN outputs, against 128 + BN for a one-CTA tile:
// with the 256 canvas rows of a step as M, every weight row is read once per
// pair instead of once per 128-row tile, and every token row half as often.
//
// Roles (192 threads in each CTA):
//   warp 0 lane 0   producer, in both CTAs: TMA copies of this CTA's halves;
//                   both signal the leader's (rank 0's) full[s] barrier
//                   (cp.async.bulk.tensor .cta_group::2), on which the leader's
//                   producer posts the transaction bytes of both halves;
//   warp 1 lane 0   MMA issuer, leader only: waits full[s], issues the four
//                   K steps of the stage for the pair, and releases stage s in
//                   both CTAs and, after the item's last stage, the accumulator
//                   in both CTAs (tcgen05.commit with a CTA mask of both);
//   warps 2..5      epilogue, in both CTAs: read this CTA's 128 TMEM lanes and
//                   run the epilogue functor on them, then arrive (locally or
//                   remotely) on the leader's tempty[acc], which counts the
//                   eight epilogue warps of the pair.
// Items (pair tiles) follow the dense schedulers in a fixed stride over the
// pairs; the epilogue functors see each CTA's half as the one-CTA item of the
// 128-row tile it holds, so they are shared with the one-CTA kernel.
// Every wait is bounded; after the roles end both CTAs meet at a cluster
// barrier (so no CTA leaves while its peer may still read its shared memory or
// arrive on its barriers), then free their tensor memory.  Every copy is an
// ordinary per-CTA copy into the issuing CTA's own shared memory.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace dgen {
namespace tc2 {

using tc::A_BYTES;
using tc::BK;
using tc::BM;

template <int BN, int STAGES, int EPI_SMEM>
struct Layout {
    static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
    static constexpr int B_HALF = BN / 2 * BK * 2;  // this CTA's B rows
    static constexpr int STAGE_BYTES = A_BYTES + B_HALF;
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    static constexpr int N_BARS = 2 * STAGES + 5;  // full[], empty[], tfull[2], tempty[2], drain
    static constexpr int SLOT_OFF = BAR_OFF + N_BARS * 8;
    static constexpr int EPI_OFF = (SLOT_OFF + 16 + 127) & ~127;
    static constexpr int SMEM_BYTES = EPI_OFF + EPI_SMEM + 1024;
    static constexpr int TMEM_COLS = 2 * BN;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier of another CTA of the cluster (shared::cluster address).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 2-D tiled copy into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (bar: shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (+)= A B^T for the pair: one 256 x N x 16 step, issued by the leader.
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on this CTA's mbarrier when every tcgen05 op of the pair issued
// so far by this thread completes.
__device__ __forceinline__ void mma_commit_pair_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Same, arriving on the mbarrier at this shared-memory offset in both CTAs of
// the pair (the commit's CTA mask 0b11).
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
            bar)
        : "memory");
}

// Dense pair scheduler over 256-row x BN tiles (x k_splits), items in the
// order of tc::DenseSched (pair rows fastest; m_tiles counts 256-row tiles).
// b_row(item, rank): the first B row of this CTA's half of the item's B tile
// (the tensor map's box is BN / 2 rows high).
struct DensePairSched : tc::DenseSched {
    template <int BN>
    __device__ __forceinline__ int b_row(int it, uint32_t rank) const {
        return n_of(it) * BN + static_cast<int>(rank) * (BN / 2);
    }
};

// The same with an MN-major B (B[n][k] stored with n contiguous, e.g. the
// embedding [V][d] as the right operand of p0_hat E): this CTA's half is BN/2
// columns, loaded as (BN/2)/64 boxes of 64 k-rows x 64 columns 8 KB apart (the
// map's box: 64 x 64), read through MN-major descriptors.
struct DensePairMNSched : DensePairSched {
    static constexpr bool kBMN = true;
};

// Pair scheduler over PairSched's RoPE tiles (BN = 2 x the box height): CTA 0
// loads the box of features f.., CTA 1 the box of their partners f + pair_off ..
struct RopePairSched : tc::PairSched {
    template <int BN>
    __device__ __forceinline__ int b_row(int it, uint32_t rank) const {
        const int per = 2 * pair_off / BN, n = n_of(it);
        return (n / per) * 2 * pair_off + (n % per) * (BN / 2) + static_cast<int>(rank) * pair_off;
    }
};

template <int BN, int STAGES, int EPI_SMEM, class Sched, class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ Sched sched, const Epi epi, const int num_kb, int* __restrict__ err) {
    using L = Layout<BN, STAGES, EPI_SMEM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SLOT_OFF);
    uint8_t* epi_smem = smem + L::EPI_OFF;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 8);  // the epilogue warps of both CTAs
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
    tc_fence_after();
    pdl_trigger();
    pdl_wait();
    const uint32_t tmem = *tmem_slot;
    const int n_items = sched.count();

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int s = 0;
            uint32_t ph = 0;
            for (int it = pair; it < n_items; it += n_pairs) {
                const int a_row = (it % sched.m_tiles) * 256 + static_cast<int>(rank) * BM;
                const int b_row = sched.template b_row<BN>(it, rank);
                int kb0, nkb;
                sched.kb_range(it, num_kb, kb0, nkb);
                bool ok = true;
                for (int kb = kb0; kb < kb0 + nkb; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, err, ERR_GEMM_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = map_to_rank(smem_u32(&full[s]), 0);
                    if (rank == 0) mbar_expect_tx(&full[s], 2 * L::STAGE_BYTES);
                    const uint32_t sa = sbase + s * L::STAGE_BYTES;
                    tma_load_2d_pair(sa, &tmA, kb * BK, a_row, fb);
                    if constexpr (Sched::kBMN) {
#pragma unroll
                        for (int c = 0; c < BN / 128; ++c)
                            tma_load_2d_pair(sa + A_BYTES + c * 8192, &tmB, b_row + 64 * c, kb * BK, fb);
                    } else {
                        tma_load_2d_pair(sa + A_BYTES, &tmB, kb * BK, b_row, fb);
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            int s = 0, lt = 0;
            uint32_t ph = 0;
            bool ok = true;
            constexpr uint32_t idesc = Sched::kBMN ? idesc_bf16_f32_bmn(2 * BM, BN) : idesc_bf16_f32(2 * BM, BN);
            for (int it = pair; ok && it < n_items; it += n_pairs, ++lt) {
                const int acc = lt & 1;
                const uint32_t aph = (lt >> 1) & 1;
                if (!mbar_wait(&tempty[acc], aph ^ 1u, err, ERR_GEMM_MMA)) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * BN;
                int kb0, nkb;
                sched.kb_range(it, num_kb, kb0, nkb);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&full[s], ph, err, ERR_GEMM_MMA)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = sbase + s * L::STAGE_BYTES;
                    const uint64_t ad = sdesc_sw128(sa), bd = sdesc_sw128(sa + A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if constexpr (Sched::kBMN)  // 16 k-rows of 128 bytes per step, 64-column blocks 8 KB apart
                            mma_bf16_pair(d, ad + 2 * k, sdesc_sw128_mn(sa + A_BYTES + k * 2048, 8192), idesc,
                                          (kb | k) != 0 ? 1u : 0u);
                        else
                            mma_bf16_pair(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(smem_u32(&empty[s]));
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(smem_u32(&tfull[acc]));
            }
            mma_commit_pair_local(smem_u32(drain));  // arrives when every MMA issued above has completed
            mbar_wait(drain, 0, err, ERR_GEMM_DRAIN);
        }
    } else {
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t tempty_leader0 = map_to_rank(smem_u32(&tempty[0]), 0);
        // this CTA's half as a one-CTA item of the 128-row tile it holds
        Sched half = sched;
        half.m_tiles = 2 * sched.m_tiles;
        int lt = 0;
        for (int it = pair; it < n_items; it += n_pairs, ++lt) {
            const int acc = lt & 1;
            const uint32_t aph = (lt >> 1) & 1;
            if (!mbar_wait(&tfull[acc], aph, err, ERR_GEMM_EPILOGUE)) break;
            tc_fence_after();
            const int mt = it % sched.m_tiles, rest = it / sched.m_tiles;
            const int it_half = 2 * mt + static_cast<int>(rank) + half.m_tiles * rest;
            epi.template run<BN>(half, it_half,
                                 tmem + acc * BN + (static_cast<uint32_t>(q * 32) << 16), q, lane, epi_smem);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(tempty_leader0 + acc * 8);
        }
    }
    tc_fence_before();
    cluster_sync();  // the pair's MMAs, copies and remote arrivals are done
    tc_fence_after();
    if (warp == 0) tmem_dealloc_pair(tmem, L::TMEM_COLS);
}

}  // namespace tc2
}  // namespace dgen
