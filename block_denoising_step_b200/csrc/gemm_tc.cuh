// Persistent warp-specialised tcgen05 GEMM core for sm_100a.
//
//   D[128 x BN] (fp32, in tensor memory) = A[128 x K] * B[BN x K]^T
//
// A and B are bf16 (KIND 0) or E4M3 (KIND 1), K-major, fetched by TMA with
// 128-byte swizzle into a STAGES-deep shared-memory ring; a k-block is one
// 128-byte swizzle row per operand row (64 bf16 or 128 E4M3 elements).  Roles (192 threads):
//   warp 0 lane 0   TMA producer: A as A_BOXES boxes of 128/A_BOXES rows whose
//                   row coordinates the scheduler gives, B as one BN-row box;
//   warp 1 lane 0   MMA issuer: 4 x tcgen05.mma (32 bytes of K each: K = 16 bf16
//                   or 32 E4M3) per k-block into one of two TMEM accumulators
//                   (BN fp32 columns each);
//   warps 2..5      epilogue: tcgen05.ld of their 32-lane quarter of the
//                   accumulator, then the epilogue functor; the next tile's
//                   MMAs run into the other accumulator meanwhile.
// Work items (output tiles) are dealt round-robin to the persistent CTAs.
// Every wait is bounded (common.cuh); on a timeout the kernel records an
// error, drains its own TMA copies and MMAs, frees its tensor memory and exits.
#pragma once

#include "common.cuh"

namespace dgen {
namespace tc {

constexpr int BM = 128;   // accumulator rows (TMEM lanes)
constexpr int BK = 64;    // one 128-byte swizzle row of bf16
constexpr int A_BYTES = BM * BK * 2;
// elements per k-block (one 128-byte row): KIND 0 bf16, KIND 1 E4M3
template <int KIND>
constexpr int bk_elems() {
    return KIND == 0 ? 64 : 128;
}

template <int BN, int STAGES, int EPI_SMEM>
struct Layout {
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256, "BN");
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    // full[], empty[], tmem_full[2], tmem_empty[2], drain, item_ready[2] (dynamic item order)
    static constexpr int N_BARS = 2 * STAGES + 7;
    static constexpr int SLOT_OFF = BAR_OFF + N_BARS * 8;
    static constexpr int ITEM_OFF = SLOT_OFF + 16;  // int stage_item[STAGES], acc_item[2]
    static constexpr int EPI_OFF = (ITEM_OFF + (STAGES + 2) * 4 + 127) & ~127;
    static constexpr int SMEM_BYTES = EPI_OFF + EPI_SMEM + 1024;  // + slack for 1024-byte alignment
    static constexpr int TMEM_COLS = (2 * BN < 32) ? 32 : 2 * BN;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// ------------------------------------------------------------------ schedulers
// coords(item, a_rows[A_BOXES], b_row): TMA row coordinates of the item's tiles.

// kb_range(item, num_kb, kb0, nkb): the k-blocks an item accumulates.  Without
// a K split every item covers all of them; with k_splits > 1, item split ks
// covers a contiguous share and its epilogue writes a partial result that the
// consumer sums in split order (deterministic).

// select(item, ma, mb, kx0): the tensor maps an item reads (default: the
// kernel's A and B maps) and the K coordinate its k-block 0 starts at.
// kStaticB: the item count and the B tile coordinates depend on no device data;
// with b_static set (B a weight matrix) B copies may start before the previous
// kernel ends.

// Dense: m_tiles x n_tiles output tiles (x k_splits); consecutive items share the B tile.
// load_b<BN>(dst, map, x, b, bar): the TMA copy(ies) of an item's B tile for
// k-block column x, b being the row coordinate coords() returned.

struct DenseSched {
    static constexpr bool kStaticB = true;  // B coordinates and item count need no device data
    static constexpr bool kBMN = false;     // B is K-major (see DenseMNSched)
    static constexpr bool kDynamic = false; // items taken in a fixed stride (see FusedExpertSched)
    int m_tiles, n_tiles;
    int k_splits = 1;
    int b_static = 0;  // 1: B is a weight no kernel writes (its copies may precede the wait)
    __device__ __forceinline__ int count() const { return m_tiles * n_tiles * k_splits; }
    __device__ __forceinline__ int m_of(int it) const { return it % m_tiles; }
    __device__ __forceinline__ int n_of(int it) const { return (it / m_tiles) % n_tiles; }
    __device__ __forceinline__ int ks_of(int it) const { return it / (m_tiles * n_tiles); }
    __device__ __forceinline__ void kb_range(int it, int num_kb, int& kb0, int& nkb) const {
        const int per = (num_kb + k_splits - 1) / k_splits;
        kb0 = ks_of(it) * per;
        nkb = max(0, min(per, num_kb - kb0));
    }
    template <int A_BOXES, int BN>
    __device__ __forceinline__ void coords(int it, int (&a)[A_BOXES], int& b) const {
#pragma unroll
        for (int j = 0; j < A_BOXES; ++j) a[j] = m_of(it) * BM + j * (BM / A_BOXES);
        b = n_of(it) * BN;
    }
    template <int BN>
    __device__ __forceinline__ void load_b(uint32_t dst, const CUtensorMap* m, int x, int b, uint32_t bar) const {
        tma_load_2d(dst, m, x, b, bar);
    }
    template <int BN>
    __device__ __forceinline__ int n_cols(int) const { return BN; }
    __device__ __forceinline__ void select(int, const CUtensorMap*&, const CUtensorMap*&, int&) const {}
    __device__ __forceinline__ void prefetch() const {}
    __device__ __forceinline__ bool item_ready(int, int*) const { return true; }
};

// Dense, with each B tile made of two half-height boxes of one 2*pair_off-row
// group: tile n takes rows g*2*pair_off + h*BN/2 .. + BN/2 - 1 and the same
// rows + pair_off (g = n / groups_per, h = n % groups_per, groups_per =
// 2*pair_off / BN).  For the QKV projection with hd = 256 and BN = 128 this
// puts the rotate-half RoPE pairs (j, j + hd/2) of a head in one tile, at
// columns c and c + BN/2.  The tensor map's box is BN/2 rows high.
struct PairSched : DenseSched {
    int pair_off = 128;
    template <int A_BOXES, int BN>
    __device__ __forceinline__ void coords(int it, int (&a)[A_BOXES], int& b) const {
#pragma unroll
        for (int j = 0; j < A_BOXES; ++j) a[j] = m_of(it) * BM + j * (BM / A_BOXES);
        const int per = 2 * pair_off / BN, n = n_of(it);
        b = (n / per) * 2 * pair_off + (n % per) * (BN / 2);
    }
    template <int BN>
    __device__ __forceinline__ void load_b(uint32_t dst, const CUtensorMap* m, int x, int b, uint32_t bar) const {
        tma_load_2d(dst, m, x, b, bar);
        tma_load_2d(dst + (BN / 2) * 128, m, x, b + pair_off, bar);
    }
};

// Dense with an MN-major B: B[n][k] is stored with n contiguous (a row-major
// [K][N] matrix, e.g. the embedding E [V][d] as the right operand of P E).  A B
// tile is BN / 64 TMA boxes of 64 k-rows x 64 n-columns (128-byte rows, 128-byte
// swizzle), 8 KB apart; the MMA reads it through MN-major descriptors (leading
// byte offset 8 KB between 64-column blocks, 2 KB per 16-element K step).
// The tensor map's box is 64 columns x 64 rows.
struct DenseMNSched : DenseSched {
    static constexpr bool kBMN = true;
    template <int BN>
    __device__ __forceinline__ void load_b(uint32_t dst, const CUtensorMap* m, int x, int b, uint32_t bar) const {
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tma_load_2d(dst + c * 8192, m, b + 64 * c, x, bar);
    }
};

// Grouped ("swap-AB") expert GEMM: A = 128 weight rows of one expert, B = a
// chunk of up to BN token rows routed to that expert.
// chunks[c] = {expert, first token row, token count, 0}; item = c * m_tiles + mt;
// the A tile of item (c, mt) is rows e * rows_per_expert + mt * 128 .. + 127.
//   gate-up: the weight rows interleave gate and up in blocks of 16, so tile mt
//     holds gate and up rows of features mt*64 .. mt*64+63 and TMEM lanes
//     32j..32j+15 / 32j+16..32j+31 hold gate / up of features mt*64 + 16j + 0..15;
//   down: tile mt holds output rows mt*128 .. mt*128+127 of W_d,e.
// A chunk whose expert id is E + j (j >= 0) belongs to the shared FFN, taken as
// pseudo-expert j: feature slice j*w .. j*w + w - 1 of the shared FFN, always
// selected with gate 1.  Its items read the second pair of maps (shared
// weights; token rows in natural order): gate-up A rows j * shared_a_stride +
// mt*128 (shared_a_stride = 2w), down K from shared_k_off * j (= w j).
struct GroupedSched {
    static constexpr bool kStaticB = false;  // items come from the routing permutation's output
    static constexpr bool kDynamic = true;   // items claimed from `queue` (see FusedExpertSched); null: fixed stride
    const int4* chunks;
    const int* n_chunks;   // device scalar
    int m_tiles;
    int rows_per_expert;   // 2w (gate-up) or d (down)
    int k_splits = 1;
    int E = 0x7fffffff;    // first pseudo-expert id of the shared FFN
    int shared_a_stride = 0;
    int shared_k_off = 0;
    CUtensorMap tmA2;        // shared FFN weights
    // token-row maps with boxes of 16 << c rows (c = 0..4): an item loads and
    // multiplies only the smallest box that holds its chunk's rows (MMA N = box)
    CUtensorMap tmBc[5], tmB2c[5];  // routed rows, shared-FFN rows
    int* queue = nullptr;           // items claimed beyond the first wave, zeroed before the launch
    __device__ __forceinline__ int count() const { return __ldg(n_chunks) * m_tiles * k_splits; }
    __device__ __forceinline__ int4 chunk(int it) const { return __ldg(&chunks[(it / k_splits) / m_tiles]); }
    __device__ __forceinline__ int mt_of(int it) const { return (it / k_splits) % m_tiles; }
    __device__ __forceinline__ int ks_of(int it) const { return it % k_splits; }
    __device__ __forceinline__ void kb_range(int it, int num_kb, int& kb0, int& nkb) const {
        const int per = (num_kb + k_splits - 1) / k_splits;
        kb0 = ks_of(it) * per;
        nkb = max(0, min(per, num_kb - kb0));
    }
    template <int A_BOXES, int BN>
    __device__ __forceinline__ void coords(int it, int (&a)[A_BOXES], int& b) const {
        const int4 ch = chunk(it);
        const int base = (ch.x < E ? ch.x * rows_per_expert : (ch.x - E) * shared_a_stride) + mt_of(it) * BM;
#pragma unroll
        for (int j = 0; j < A_BOXES; ++j) a[j] = base + j * (BM / A_BOXES);
        b = ch.y;
    }
    template <int BN>
    __device__ __forceinline__ void load_b(uint32_t dst, const CUtensorMap* m, int x, int b, uint32_t bar) const {
        tma_load_2d(dst, m, x, b, bar);
    }
    __device__ __forceinline__ static int box_class(int rows) {
        return rows <= 16 ? 0 : rows <= 32 ? 1 : rows <= 64 ? 2 : rows <= 128 ? 3 : 4;
    }
    template <int BN>
    __device__ __forceinline__ int n_cols(int it) const { return min(BN, 16 << box_class(chunk(it).z)); }
    __device__ __forceinline__ void select(int it, const CUtensorMap*& ma, const CUtensorMap*& mb, int& kx0) const {
        const int4 ch = chunk(it);
        const int c = box_class(ch.z);
        if (ch.x >= E) {
            ma = &tmA2;
            mb = &tmB2c[c];
            kx0 = (ch.x - E) * shared_k_off;
        } else {
            mb = &tmBc[c];
        }
    }
    __device__ __forceinline__ void prefetch() const {
#pragma unroll
        for (int c = 0; c < 5; ++c) prefetch_tmap(&tmBc[c]);
        if (E != 0x7fffffff) {
            prefetch_tmap(&tmA2);
#pragma unroll
            for (int c = 0; c < 5; ++c) prefetch_tmap(&tmB2c[c]);
        }
    }
    __device__ __forceinline__ bool item_ready(int, int*) const { return true; }
    static constexpr bool kBMN = false;
};

// Both grouped expert GEMMs of a layer in one persistent launch: items
// [0, n_gu) are the gate-up items of the chunk list (gu, item = c * m_gu + mt),
// items [n_gu, n_gu + n_dn) its down items (dn).  Items are taken dynamically:
// CTA b starts with item b, then claims the next untaken item from a global
// counter (`queue`, zeroed before the launch), so an SM that drew small items
// takes more of them and the launch ends with at most one item of imbalance.
// Items are claimed in increasing order, so every gate-up item is claimed (by
// a running CTA) before any down item.
// A down item of chunk c reads the gated activations of c's rows, which the
// gate-up items of c write: each of their four epilogue warps adds 1 to
// ready[c] after its stores (made visible to the async proxy, then released),
// and the producer waits (bounded; acquire, then a proxy fence) until ready[c]
// reaches 4 m_gu before loading the item's B tiles.  Gate-up items wait for
// nothing, so every down item's wait ends as long as every CTA of the launch
// runs, which a grid of at most one CTA per SM ensures.
struct FusedExpertSched {
    static constexpr bool kStaticB = false;
    static constexpr bool kBMN = false;
    static constexpr bool kDynamic = true;
    int* queue;                  // items claimed beyond the first wave, zeroed before the launch
                                 // (null: fixed stride, item b + j gridDim.x)
    GroupedSched gu, dn;
    CUtensorMap tmA_gu, tmA_dn;  // routed gate-up / down weights
    int kb_gu, kb_dn;            // k-blocks of a gate-up / down item
    int* ready;                  // [chunks], zeroed before the launch
    __device__ __forceinline__ int n_gu() const { return __ldg(gu.n_chunks) * gu.m_tiles; }
    __device__ __forceinline__ int count() const { return n_gu() + __ldg(dn.n_chunks) * dn.m_tiles; }
    __device__ __forceinline__ bool is_gu(int it) const { return it < n_gu(); }
    __device__ __forceinline__ void kb_range(int it, int, int& kb0, int& nkb) const {
        kb0 = 0;
        nkb = is_gu(it) ? kb_gu : kb_dn;
    }
    template <int A_BOXES, int BN>
    __device__ __forceinline__ void coords(int it, int (&a)[A_BOXES], int& b) const {
        const int g = n_gu();
        if (it < g)
            gu.template coords<A_BOXES, BN>(it, a, b);
        else
            dn.template coords<A_BOXES, BN>(it - g, a, b);
    }
    template <int BN>
    __device__ __forceinline__ void load_b(uint32_t dst, const CUtensorMap* m, int x, int b, uint32_t bar) const {
        tma_load_2d(dst, m, x, b, bar);
    }
    template <int BN>
    __device__ __forceinline__ int n_cols(int it) const {
        const int g = n_gu();
        return it < g ? gu.template n_cols<BN>(it) : dn.template n_cols<BN>(it - g);
    }
    __device__ __forceinline__ void select(int it, const CUtensorMap*& ma, const CUtensorMap*& mb, int& kx0) const {
        const int g = n_gu();
        if (it < g) {
            ma = &tmA_gu;
            gu.select(it, ma, mb, kx0);
        } else {
            ma = &tmA_dn;
            dn.select(it - g, ma, mb, kx0);
        }
    }
    __device__ __forceinline__ void prefetch() const {
        prefetch_tmap(&tmA_gu);
        prefetch_tmap(&tmA_dn);
        gu.prefetch();
        dn.prefetch();
    }
    __device__ __forceinline__ bool item_ready(int it, int* err) const {
        const int g = n_gu();
        if (it < g) return true;
        const int c = (it - g) / dn.m_tiles;
        const int target = 4 * gu.m_tiles;
        if (ld_acquire_s32(&ready[c]) < target) {
            const uint64_t t0 = globaltimer_ns();
            uint32_t nap = 64;
            while (ld_acquire_s32(&ready[c]) < target) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    if (err) atomicExch(err, ERR_GEMM_READY);
                    return false;
                }
                __nanosleep(nap);
                nap = min(nap * 2, 2048u);
            }
        }
        fence_proxy_async_global();
        return true;
    }
};

// ------------------------------------------------------------------ kernel

template <int BN, int STAGES, int A_BOXES, int EPI_SMEM, class Sched, class Epi, int KIND = 0>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ Sched sched,
                const Epi epi, const int num_kb, int* __restrict__ err) {
    using L = Layout<BN, STAGES, EPI_SMEM>;
    constexpr int BKE = bk_elems<KIND>();
    constexpr int A_BOX_BYTES = A_BYTES / A_BOXES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* titem = drain + 1;  // acc_item[a] published (dynamic item order)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SLOT_OFF);
    volatile int* stage_item = reinterpret_cast<volatile int*>(smem + L::ITEM_OFF);
    volatile int* acc_item = stage_item + STAGES;
    uint8_t* epi_smem = smem + L::EPI_OFF;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
            mbar_init(&titem[a], 1);
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
    // The prologue above overlapped the previous kernel's tail.  Every thread
    // but the producer waits for that kernel here; the producer first starts the
    // B loads (weights, which no kernel writes) of its first item's first stages
    // when the scheduler says they do not depend on the previous kernel.
    pdl_trigger();
    const bool producer = warp == 0 && lane == 0;
    if (!producer) pdl_wait();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int pre = 0;  // stages of the first item whose B copy is already in flight
            if constexpr (Sched::kStaticB) {
                const int it0 = blockIdx.x;
                if (sched.b_static && it0 < sched.count()) {
                    int ar[A_BOXES], br, kb0, nkb;
                    sched.template coords<A_BOXES, BN>(it0, ar, br);
                    sched.kb_range(it0, num_kb, kb0, nkb);
                    pre = min(STAGES, nkb);
                    for (int p = 0; p < pre; ++p) {
                        mbar_expect_tx(&full[p], L::STAGE_BYTES);
                        sched.template load_b<BN>(sbase + p * L::STAGE_BYTES + A_BYTES, &tmB, (kb0 + p) * BKE, br,
                                                  smem_u32(&full[p]));
                    }
                }
            }
            pdl_wait();
            sched.prefetch();
            const int n_items = sched.count();
            int s = 0;
            uint32_t ph = 0, pending = 0, fill_ph = 0;
            bool ok = true;
            bool first = true;
            for (int it = blockIdx.x; ok && it < n_items; first = false) {
                int ar[A_BOXES], br, kb0, nkb, kx0 = 0;
                const CUtensorMap* ma = &tmA;
                const CUtensorMap* mb = &tmB;
                if (!sched.item_ready(it, err)) {
                    ok = false;
                    break;
                }
                sched.template coords<A_BOXES, BN>(it, ar, br);
                sched.select(it, ma, mb, kx0);
                sched.kb_range(it, num_kb, kb0, nkb);
                const int nc = sched.template n_cols<BN>(it);  // B rows this item loads
                for (int kb = kb0; kb < kb0 + nkb; ++kb) {
                    const bool b_issued = first && kb - kb0 < pre;  // B started before the wait
                    if (!mbar_wait(&empty[s], ph ^ 1u, err, ERR_GEMM_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    pending &= ~(1u << s);
                    const uint32_t fb = smem_u32(&full[s]);
                    if constexpr (Sched::kDynamic) stage_item[s] = it;  // read by the MMA warp after full[s]
                    if (!b_issued) mbar_expect_tx(&full[s], A_BYTES + nc * (BK * 2));
                    const uint32_t sa = sbase + s * L::STAGE_BYTES;
#pragma unroll
                    for (int j = 0; j < A_BOXES; ++j) tma_load_2d(sa + j * A_BOX_BYTES, ma, kx0 + kb * BKE, ar[j], fb);
                    if (!b_issued) sched.template load_b<BN>(sa + A_BYTES, mb, kx0 + kb * BKE, br, fb);
                    pending |= 1u << s;
                    fill_ph = (fill_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if constexpr (Sched::kDynamic)
                    it = sched.queue ? static_cast<int>(gridDim.x) + atomicAdd(sched.queue, 1) : it + gridDim.x;
                else
                    it += gridDim.x;
            }
            if constexpr (Sched::kDynamic) {
                // no item left: a marker stage (item -1, no copy) tells the MMA warp,
                // and through it the epilogue warps, to stop
                if (ok && mbar_wait(&empty[s], ph ^ 1u, err, ERR_GEMM_PRODUCER)) {
                    stage_item[s] = -1;
                    mbar_arrive(&full[s]);
                }
            }
            if (!ok) {  // let our own copies land before the CTA goes away
                for (int j = 0; j < STAGES; ++j)
                    if ((pending >> j) & 1u) mbar_wait(&full[j], (fill_ph >> j) & 1u, err, ERR_GEMM_DRAIN);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            if constexpr (Sched::kDynamic) {
                // items in the order the producer claimed them: the first stage of each
                // names it (stage_item), and acc_item[acc] + titem[acc] pass it on to
                // the epilogue warps; item -1 ends the launch
                int s = 0, lt = 0;
                uint32_t ph = 0;
                bool ok = true;
                for (;; ++lt) {
                    const int acc = lt & 1;
                    const uint32_t aph = (lt >> 1) & 1;
                    if (!mbar_wait(&tempty[acc], aph ^ 1u, err, ERR_GEMM_MMA)) break;
                    if (!mbar_wait(&full[s], ph, err, ERR_GEMM_MMA)) break;
                    const int it = stage_item[s];
                    acc_item[acc] = it;
                    mbar_arrive(&titem[acc]);
                    if (it < 0) break;
                    tc_fence_after();
                    const uint32_t d = tmem + acc * BN;
                    const uint32_t idesc = KIND == 0 ? idesc_bf16_f32(BM, sched.template n_cols<BN>(it))
                                                     : idesc_e4m3_f32(BM, sched.template n_cols<BN>(it));
                    int kb0, nkb;
                    sched.kb_range(it, num_kb, kb0, nkb);
                    for (int kb = 0; kb < nkb; ++kb) {
                        if (kb > 0 && !mbar_wait(&full[s], ph, err, ERR_GEMM_MMA)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = sbase + s * L::STAGE_BYTES;
                        const uint64_t ad = sdesc_sw128(sa), bd = sdesc_sw128(sa + A_BYTES);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            if constexpr (KIND == 0)
                                mma_bf16_ss(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                            else
                                mma_e4m3_ss(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                        }
                        mma_commit(smem_u32(&empty[s]));
                        if (++s == STAGES) {
                            s = 0;
                            ph ^= 1u;
                        }
                    }
                    if (!ok) break;
                    mma_commit(smem_u32(&tfull[acc]));
                }
            } else {
                const int n_items = sched.count();
                int s = 0, lt = 0;
                uint32_t ph = 0;
                bool ok = true;
                for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++lt) {
                    const int acc = lt & 1;
                    const uint32_t aph = (lt >> 1) & 1;
                    if (!mbar_wait(&tempty[acc], aph ^ 1u, err, ERR_GEMM_MMA)) break;
                    tc_fence_after();
                    const uint32_t d = tmem + acc * BN;
                    const uint32_t idesc = KIND == 0 ? (Sched::kBMN ? idesc_bf16_f32_bmn(BM, sched.template n_cols<BN>(it))
                                                                    : idesc_bf16_f32(BM, sched.template n_cols<BN>(it)))
                                                     : idesc_e4m3_f32(BM, sched.template n_cols<BN>(it));
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
                        for (int k = 0; k < 4; ++k) {  // four 32-byte K steps per 128-byte row
                            if constexpr (KIND == 0 && Sched::kBMN) {
                                // MN-major B: 16 k-rows of 128 bytes per step, 64-column blocks 8 KB apart
                                mma_bf16_ss(d, ad + 2 * k, sdesc_sw128_mn(sa + A_BYTES + k * 2048, 8192), idesc,
                                            (kb | k) != 0 ? 1u : 0u);
                            } else if constexpr (KIND == 0) {
                                mma_bf16_ss(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                            } else {
                                mma_e4m3_ss(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                            }
                        }
                        mma_commit(smem_u32(&empty[s]));
                        if (++s == STAGES) {
                            s = 0;
                            ph ^= 1u;
                        }
                    }
                    if (!ok) break;
                    mma_commit(smem_u32(&tfull[acc]));
                }
            }
            mma_commit(smem_u32(drain));  // arrives when every MMA issued above has completed
            mbar_wait(drain, 0, err, ERR_GEMM_DRAIN);
        }
    } else {
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        if constexpr (Sched::kDynamic) {
            for (int lt = 0;; ++lt) {
                const int acc = lt & 1;
                const uint32_t aph = (lt >> 1) & 1;
                if (!mbar_wait(&titem[acc], aph, err, ERR_GEMM_EPILOGUE)) break;
                const int it = acc_item[acc];
                if (it < 0) break;
                if (!mbar_wait(&tfull[acc], aph, err, ERR_GEMM_EPILOGUE)) break;
                tc_fence_after();
                epi.template run<BN>(sched, it, tmem + acc * BN + (static_cast<uint32_t>(q * 32) << 16), q, lane,
                                     epi_smem);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
            }
        } else {
            const int n_items = sched.count();
            int lt = 0;
            for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++lt) {
                const int acc = lt & 1;
                const uint32_t aph = (lt >> 1) & 1;
                if (!mbar_wait(&tfull[acc], aph, err, ERR_GEMM_EPILOGUE)) break;
                tc_fence_after();
                epi.template run<BN>(sched, it, tmem + acc * BN + (static_cast<uint32_t>(q * 32) << 16), q, lane,
                                     epi_smem);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace tc
}  // namespace dgen
