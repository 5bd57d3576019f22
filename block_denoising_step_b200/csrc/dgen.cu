// dgen: host engine and C ABI of the block denoising step (see include/dgen.h).
//
// One handle = one model on one device.  The handle records the caller's weight
// pointers, owns the KV cache, the canvas state and all scratch, and enqueues
// every step of the path as CUDA kernels on its stream.  Per decoder layer
// (10 launches; RMSNorms fused into the kernel that produces their input):
//   QKV GEMM (+RoPE, scatter to Q / KV cache) -> attention (+ split combine)
//   -> O GEMM (K-split partials) -> residual add + RMSNorm -> router GEMM
//   -> routing (top-k + gates, permutation, chunk list, row gather)
//   -> grouped gate-up GEMM (+GELU * up; the shared FFN as pseudo-experts)
//   -> grouped down GEMM (* gate) -> combine + residual + next RMSNorm;
// then the tied LM head GEMM whose epilogue reduces each row to softmax
// statistics; the sampler reads only those statistics.  The decoder pass is
// captured once per prompt length into a CUDA graph and replayed.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <utility>
#include <vector>

#include "dgen.h"
#ifdef DGEN_PROBES
#include "dgen_probe.h"
#endif
#include "attention.cuh"
#include "attention_tc.cuh"
#include "eb_sampler.cuh"
#include "common.cuh"
#include "epilogues.cuh"
#include "gemm_pair.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"

using namespace dgen;

namespace {

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

bool load_encode() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    return g_encode != nullptr;
}

// 2-D bf16 tensor [rows][cols] (row-major), box = 64 columns x box_rows rows,
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    if (!g_encode || base == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) || (cols * 2) % 16 != 0 ||
        rows == 0 || box_rows == 0 || box_rows > 256)
        return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte tensor [rows][cols] (E4M3 values), box = 128 columns x box_rows rows,
// 128-byte swizzle: the same 128-byte rows as the bf16 maps.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    if (!g_encode || base == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) || cols % 16 != 0 || rows == 0 ||
        box_rows == 0 || box_rows > 256)
        return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {128, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMM launch

template <int BN>
constexpr int stages_for() {
    return BN <= 64 ? 8 : (BN == 128 ? 6 : 4);
}


// Raise a kernel's dynamic shared-memory limit to at least `bytes` on a
// device (kept per (kernel, device) and only ever raised: a kernel whose
// dynamic size depends on the shape must not be capped by an earlier, smaller
// launch).  Keyed on the kernel's address: instantiations that differ only in
// tile size share a function type.
std::mutex g_attr_mu;
std::map<std::pair<const void*, int>, int> g_attr_bytes;

template <class K>
void set_smem_attr_once(K kern, int bytes, int dev) {
    const void* f = reinterpret_cast<const void*>(kern);
    std::lock_guard<std::mutex> lock(g_attr_mu);
    int& cur = g_attr_bytes[{f, dev}];
    if (bytes > cur) {
        cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        cur = bytes;
    }
}

// Launch with the programmatic-stream-serialization attribute: the kernel may be
// scheduled while its predecessor drains; each kernel waits (griddepcontrol)
// before touching memory the predecessor writes.
std::atomic<bool> g_pdl{true};  // cleared by DGEN_FLAG_NO_PDL on any handle (process-wide)

template <typename... KArgs, typename... Args>
cudaError_t launch_ex(cudaStream_t st, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = g_pdl.load(std::memory_order_relaxed) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// KIND 0: bf16 operands; 1: E4M3 operands (K counted in elements either way).
template <int BN, int A_BOXES, class Sched, class Epi, int KIND = 0>
int launch_gemm(cudaStream_t st, int dev, int* err, const CUtensorMap& ta, const CUtensorMap& tb, const Sched& sc,
                const Epi& ep, int K, int grid, int64_t* counter) {
    constexpr int ST = stages_for<BN>();
    constexpr int BKE = tc::bk_elems<KIND>();
    using L = tc::Layout<BN, ST, 0>;
    auto kern = tc::gemm_kernel<BN, ST, A_BOXES, 0, Sched, Epi, KIND>;
    set_smem_attr_once(kern, L::SMEM_BYTES, dev);
    if (grid < 1) grid = 1;
    const cudaError_t e = launch_ex(st, kern, dim3(grid), dim3(192), L::SMEM_BYTES, ta, tb, sc, ep,
                                    (K + BKE - 1) / BKE, err);
    if (counter) ++*counter;
    return e == cudaSuccess ? DGEN_OK : DGEN_ECUDA;
}

// The same on CTA pairs (gemm_pair.cuh): `pairs` pairs of CTAs, each pair one
// 256 x BN tile at a time; the B map's box is BN / 2 rows high.
template <int BN, class Sched, class Epi>
int launch_gemm_pair(cudaStream_t st, int dev, int* err, const CUtensorMap& ta, const CUtensorMap& tb,
                     const Sched& sc, const Epi& ep, int K, int pairs, int64_t* counter) {
    constexpr int ST = BN == 256 ? 6 : 8;
    using L = tc2::Layout<BN, ST, 0>;
    auto kern = tc2::gemm_pair_kernel<BN, ST, 0, Sched, Epi>;
    set_smem_attr_once(kern, L::SMEM_BYTES, dev);
    if (pairs < 1) pairs = 1;
    const cudaError_t e = launch_ex(st, kern, dim3(2 * pairs), dim3(192), L::SMEM_BYTES, ta, tb, sc, ep,
                                    (K + tc::BK - 1) / tc::BK, err);
    if (counter) ++*counter;
    return e == cudaSuccess ? DGEN_OK : DGEN_ECUDA;
}

struct LayerMaps {
    CUtensorMap wqkv, wo, wr, wgu, wd, wsgu, wsd;
    CUtensorMap kc, vc;  // this layer's K / V cache rows, 64-row boxes (tcgen05 attention)
    CUtensorMap wqkv_pair;  // W_qkv with 64-row boxes (PairSched QKV tiles, hd = 256)
    CUtensorMap wgu8, wd8, wsgu8, wsd8;  // E4M3 expert / shared-FFN weights (expert_fp8)
};

}  // namespace

// ------------------------------------------------------------------ handle

struct dgen_handle {
    dgen_config cfg{};
    const uint16_t* embed = nullptr;
    const uint16_t* final_norm = nullptr;
    std::vector<dgen_layer_weights> layers;
    std::vector<LayerMaps> maps;
    cudaStream_t stream = nullptr;
    int device = 0, num_sms = 148;
    int S_max = 0, rows_c = 0, rows_max = 0, bn_router = 16, max_splits = kMaxAttnSplits, max_chunks = 0;
    int n_shared_parts = 0;  // shared FFN feature slices of width w (pseudo-experts)
    int P = -1;
    std::vector<int> kv_P;
    int64_t launches = 0;
    cudaError_t last_launch = cudaSuccess;
    std::vector<void*> allocs;

    int32_t* tok = nullptr;
    uint8_t* committed = nullptr;
    bf16* kc = nullptr;
    bf16* vc = nullptr;
    size_t kv_layer = 0;
    float* h = nullptr;
    bf16* xn = nullptr;
    bf16* q = nullptr;
    bf16* attn = nullptr;
    float* part_o = nullptr;
    float* part_lse = nullptr;
    float* rlogits = nullptr;
    float* qkv_parts = nullptr;   // QKV K-split partials [qkv_parts_rows][(Hq+2Hkv) hd]
    float* oparts = nullptr;      // O-projection K-split partials [oparts_rows][d]
    size_t qkv_parts_rows = 0, oparts_rows = 0;
    int* topk_id = nullptr;
    float* topk_gate = nullptr;
    int* perm_tok = nullptr;
    float* perm_gate = nullptr;
    int* inv = nullptr;
    int4* chunks = nullptr;
    int* n_chunks = nullptr;
    int* touched = nullptr;  // [L] experts routed to in the last pass, per layer
    // routing-kernel words zeroed by each pass's embedding kernel: [L] grid-barrier
    // counters, then [L][256] rows reserved per expert
    unsigned int* barriers = nullptr;
    // [L] grid-barrier counters, [L][256] rows reserved per expert, [L][max_chunks]
    // gate-up tiles finished per chunk (fused expert launch), [L][3] items claimed
    // (the fused expert launch, or the separate gate-up and down launches)
    int route_words() const { return cfg.n_layers * (260 + max_chunks); }
    int* route_tot(int l) const { return reinterpret_cast<int*>(barriers + cfg.n_layers) + l * 256; }
    int* ready_l(int l) const {
        return reinterpret_cast<int*>(barriers + cfg.n_layers) + cfg.n_layers * 256 + l * max_chunks;
    }
    // which: 0 the fused expert launch, 1 the separate gate-up launch, 2 the separate down launch
    int* queue_l(int l, int which = 0) const {
        return reinterpret_cast<int*>(barriers + cfg.n_layers) + cfg.n_layers * (256 + max_chunks) + 3 * l + which;
    }
    bf16* xperm = nullptr;
    bf16* act = nullptr;
    float* yperm = nullptr;
    bf16* act_sh = nullptr;
    float* y_sh = nullptr;
    float* pmax = nullptr;
    float* psum = nullptr;
    float* pent = nullptr;   // per-(row, vocab tile) entropy term of the LM head's statistics
    int* parg = nullptr;
    float* conf = nullptr;
    int* argmax = nullptr;
    int* eb_prev_argmax = nullptr;  // entropy-bounded sampler: argmax canvas of its previous step
    uint8_t* eb_done = nullptr;     // entropy-bounded sampler: canvas finished in this block [B]
    uint8_t* host_flags = nullptr;  // pinned host copy of eb_done for the block loop [B]
    int blocks_done = 0;            // canvases appended to the cache since the prompt (Philox position offset)
    unsigned int route_barrier_extra = 0;  // test hook: raises the routing barrier's target
    float2* rope = nullptr;
    float* inv_tau = nullptr;  // [2]: log2(e)/tau of the step ([0]) and of the given-logits
                               // entropy-bounded path ([1])
    int* err = nullptr;
    int32_t* prompt_buf = nullptr;

    CUtensorMap map_xn_a{}, map_attn_a{}, map_embed_b{};
    CUtensorMap map_embed_b128{};  // the embedding with 128-row boxes (LM head on CTA pairs)
    CUtensorMap map_q_attn{};  // queries [B Hq n_q][hd] of either pass (up to B Hq max(C, prompt_max) rows), 128-row boxes
    // the same token-row matrices with boxes of 16 << c rows (grouped GEMM box classes)
    CUtensorMap map_xperm_c[5]{}, map_act_c[5]{}, map_xn_c[5]{}, map_actsh_c[5]{};
    // E4M3 experts (cfg.expert_fp8): quantized weights of all layers with their
    // row scales, quantized token rows / activations with theirs, and maps
    bool fp8 = false;
    int wpad = 0;  // the shared FFN's down K slices padded to whole 128-element k-blocks
    uint8_t *wgu8 = nullptr, *wd8 = nullptr, *wsgu8 = nullptr, *wsd8 = nullptr;
    float *sgu = nullptr, *sd = nullptr, *ssgu = nullptr, *ssd = nullptr;
    uint8_t *xperm8 = nullptr, *xn8 = nullptr, *act8 = nullptr, *actsh8 = nullptr;
    float *sxperm8 = nullptr, *sxn8 = nullptr, *sact8 = nullptr, *sactsh8 = nullptr;
    CUtensorMap map_xperm8_c[5]{}, map_xn8_c[5]{}, map_act8_c[5]{}, map_actsh8_c[5]{};
    // self-conditioning (cfg.self_cond_width > 0): z = FFW(p0_hat E) for the next pass
    bool sc = false;
    const uint16_t* sc_norm = nullptr;
    float* sc_logits = nullptr;  // [rows_c][V] fp32, the LM head's output when the caller stores none
    bf16* sc_p = nullptr;        // p0_hat [rows_c][V]
    float* sc_u = nullptr;       // K-split partials of p0_hat E [sc_ks][rows_c][d]
    bf16* sc_n = nullptr;        // RMSNorm(u) [rows_c][d]
    bf16* sc_act = nullptr;      // FFW activations [rows_c][w_sc]
    float* sc_z = nullptr;       // K-split partials of z [sc_kz][rows_c][d]
    int sc_ks = 1, sc_kz = 1, sc_bn_pe = 256, sc_bn_gu = 128, sc_slices = 1;
    bool sc_pairs = false;  // p0_hat E on CTA pairs (d a multiple of 256)
    CUtensorMap map_sc_p{}, map_embed_mn{}, map_sc_n{}, map_sc_wgu{}, map_sc_act{}, map_sc_wd{};
    size_t sc_z_bytes() const { return static_cast<size_t>(sc_kz) * rows_c * cfg.d_model * sizeof(float); }

    // per-kernel-class event timing (dgen_set_timing)
    struct TimedPair {
        cudaEvent_t a, b;
        int cls;
    };
    int32_t* cap_ids = nullptr;      // dgen_capture_routing
    float* cap_logits = nullptr;
    float* cap_h = nullptr;          // dgen_capture_residual
    const int32_t* force_prompt = nullptr;  // dgen_force_routing
    const int32_t* force_canvas = nullptr;
    uint32_t timing_mask = 0;
    std::vector<TimedPair> timed;
    // dgen_set_tuning overrides (0 = automatic)
    int tune_chunk = 0, tune_attn_splits = 0, tune_router_splits = 0, tune_qkv_splits = 0, tune_attn_kernel = 0;
    int tune_separate_experts = 0;  // 1: gate-up and down as two launches (measurement)
    int tune_static_items = 0;      // 1: the fused expert launch takes its items in a fixed stride (measurement)
    int tune_chunk_order = 0;       // routed chunks: 0 automatic, 1 expert id order, 2 largest expert first
    // dense GEMMs on CTA pairs: 0 the LM head and p0_hat E (automatic), 1 none,
    // 2 also the QKV and O projections (measured slower: short K, see dgen.h)
    int tune_pairs = 0;
    // captured decoder pass (dgen_denoise_step without logits / capture)
    bool use_graph = true;
    cudaGraphExec_t graph = nullptr;
    int graph_P = -1, warm_P = -1;
    const int32_t* graph_force = nullptr;  // canvas routing forced when the graph was captured
    uint32_t graph_mask = 0;
    int64_t graph_launches = 0;
    std::vector<TimedPair> graph_pairs;
    std::vector<cudaEvent_t> ev_pool;
    double t_ms[DGEN_K_CLASSES] = {};
    int64_t t_n[DGEN_K_CLASSES] = {};
    cudaEvent_t take_event() {
        if (!ev_pool.empty()) {
            cudaEvent_t e = ev_pool.back();
            ev_pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        cudaEventCreate(&e);
        return e;
    }

    template <class T>
    bool alloc(T** p, size_t n) {
        void* v = nullptr;
        if (cudaMalloc(&v, std::max<size_t>(n, 1) * sizeof(T)) != cudaSuccess) return false;
        allocs.push_back(v);
        *p = static_cast<T*>(v);
        return true;
    }
    // the router's partial-logit buffer holds rlogits_rows x E floats
    size_t rlogits_rows = 0;
    int router_max_splits(int rows) const { return std::max<int>(1, static_cast<int>(rlogits_rows / rows)); }
    bf16* kc_l(int l) const { return kc + kv_layer * l; }
    bf16* vc_l(int l) const { return vc + kv_layer * l; }
};

namespace {

constexpr int kBNs[4] = {32, 64, 128, 256};

// Records a CUDA event pair on the handle's stream around the launches in its
// scope when the class is enabled in the timing mask.
struct Timed {
    dgen_handle* h;
    int cls;
    cudaEvent_t a = nullptr;
    // While the stream is being captured the records become graph nodes that
    // record the events on every replay (cudaEventRecordExternal).
    static void record(cudaEvent_t e, cudaStream_t st) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaStreamIsCapturing(st, &cs);
        if (cs == cudaStreamCaptureStatusActive)
            cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
        else
            cudaEventRecord(e, st);
    }
    Timed(dgen_handle* h_, int c) : h(h_), cls(c) {
        if ((h->timing_mask >> c) & 1u) {
            a = h->take_event();
            record(a, h->stream);
        }
    }
    ~Timed() {
        if (a) {
            cudaEvent_t b = h->take_event();
            record(b, h->stream);
            h->timed.push_back({a, b, cls});
        }
    }
};

// Launch on the handle's stream (programmatic serialization); the status is
// read back by check_launch.
template <typename... KArgs, typename... Args>
void launch_h(dgen_handle* h, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, Args... args) {
    h->last_launch = launch_ex(h->stream, kern, grid, block, smem, args...);
}

int check_launch(dgen_handle* h) {
    ++h->launches;
    return h->last_launch == cudaSuccess ? DGEN_OK : DGEN_ECUDA;
}

#define DGEN_TRY(...)                    \
    do {                                 \
        const int _rc = (__VA_ARGS__);   \
        if (_rc != DGEN_OK) return _rc;  \
    } while (0)

// Token-chunk width of the grouped expert GEMMs: the smallest of {32, 64, 128,
// 256} holding 3x the mean rows per expert.  Routing is uneven (the routed
// experts get several times the mean), and each extra chunk of an expert
// streams its weight tile through shared memory again.
// Token-chunk width (the grouped GEMMs' BN) for `mean_rows` routed rows per
// expert.  Each chunk item loads only the box class that holds its rows, so a
// wide chunk costs nothing for small experts and saves weight re-reads for
// popular ones; at up to 32 rows per expert on average (the single-canvas
// workloads, where routing concentrates on a few popular experts) 128 measured
// best, above that the smallest width >= 3x the mean.
int pick_chunk(double mean_rows) {
    if (mean_rows <= 32.0) return 128;
    for (int bn : kBNs)
        if (bn >= 3.0 * mean_rows) return bn;
    return 256;
}

// x = E[tok] (+ z, the self-conditioning state, for a canvas pass with z set)
// and the first layer's attention-normed input, fused.
int embed(dgen_handle* h, const int32_t* tok, int rows, const float* z = nullptr) {
    launch_h(h, embed_norm_kernel, rows, 128, 0, tok, h->embed, h->h,
             static_cast<const uint16_t*>(h->layers[0].attn_norm), h->xn, rows, h->cfg.d_model, h->cfg.vocab,
             h->cfg.rms_eps, h->barriers, h->route_words(), z, h->sc_kz,
             static_cast<size_t>(h->rows_c) * h->cfg.d_model);
    return check_launch(h);
}

// gain of the norm that follows layer l's last kernel: the next layer's
// attention norm, or the final norm after the last layer
const void* next_norm_of(const dgen_handle* h, int l) {
    return l + 1 < h->cfg.n_layers ? h->layers[l + 1].attn_norm : h->final_norm;
}

int attention(dgen_handle* h, int l, int n_q, int S, int pos0, bool causal) {
    const dgen_config& c = h->cfg;
    AttnArgs a;
    a.q = h->q;
    a.k = h->kc_l(l);
    a.v = h->vc_l(l);
    a.o = h->attn;
    a.part_o = h->part_o;
    a.part_lse = h->part_lse;
    a.B = c.batch;
    a.Hq = c.n_q_heads;
    a.Hkv = c.n_kv_heads;
    a.n_q = n_q;
    a.S = S;
    a.S_max = h->S_max;
    a.q_pos0 = pos0;
    a.causal = causal ? 1 : 0;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.head_dim)));
    if (h->tune_attn_kernel == 0) {
        // tcgen05 kernel: 128-row query tiles, one CTA per SM; about one wave of
        // key splits, each at least two 64-key tiles (causal: each CTA's keys end
        // at its last query's position)
        const int q_tiles = (n_q + attn_tc::BQ - 1) / attn_tc::BQ;
        const int base = q_tiles * c.n_q_heads * c.batch;
        int splits = std::max(1, h->num_sms / std::max(1, base));
        if (h->tune_attn_splits > 0) splits = h->tune_attn_splits;
        splits = std::min(splits, h->max_splits);
        splits = std::min(splits, std::max(1, S / 128));
        int kps = ((S + splits - 1) / splits + 63) / 64 * 64;
        splits = (S + kps - 1) / kps;
        a.n_splits = splits;
        a.keys_per_split = kps;
        const dim3 grid(q_tiles, c.n_q_heads, c.batch * splits);
        const LayerMaps& m = h->maps[l];
        switch (c.head_dim) {
            case 64: {
                auto kern = attention_tc_kernel<64>;
                set_smem_attr_once(kern, attn_tc::Layout<64>::SMEM_BYTES, h->device);
                launch_h(h, kern, grid, attn_tc::kThreads, attn_tc::Layout<64>::SMEM_BYTES, h->map_q_attn, m.kc, m.vc, a, h->err);
                break;
            }
            case 128: {
                auto kern = attention_tc_kernel<128>;
                set_smem_attr_once(kern, attn_tc::Layout<128>::SMEM_BYTES, h->device);
                launch_h(h, kern, grid, attn_tc::kThreads, attn_tc::Layout<128>::SMEM_BYTES, h->map_q_attn, m.kc, m.vc, a, h->err);
                break;
            }
            default: {
                auto kern = attention_tc_kernel<256>;
                set_smem_attr_once(kern, attn_tc::Layout<256>::SMEM_BYTES, h->device);
                launch_h(h, kern, grid, attn_tc::kThreads, attn_tc::Layout<256>::SMEM_BYTES, h->map_q_attn, m.kc, m.vc, a, h->err);
                break;
            }
        }
        DGEN_TRY(check_launch(h));
        if (splits > 1) {
            const int rows = c.batch * c.n_q_heads * n_q;
            switch (c.head_dim) {
                case 64: launch_h(h, attention_combine_kernel<64>, (rows + 7) / 8, 256, 0, a); break;
                case 128: launch_h(h, attention_combine_kernel<128>, (rows + 7) / 8, 256, 0, a); break;
                default: launch_h(h, attention_combine_kernel<256>, (rows + 7) / 8, 256, 0, a); break;
            }
            DGEN_TRY(check_launch(h));
        }
        return DGEN_OK;
    }
    const int q_tiles = (n_q + 63) / 64;
    const int base = q_tiles * c.n_q_heads * c.batch;
    int splits = 1, kps = S;
    if (!causal) {
        // about one wave: (SMs x CTAs that fit per SM) / CTAs per split, rounded down
        const int smem_need = 5 * 64 * c.head_dim * 2;
        const int per_sm = std::max(1, std::min(4, (227 * 1024) / (smem_need + 1024)));
        splits = std::max(1, (h->num_sms * per_sm) / std::max(1, base));
        if (h->tune_attn_splits > 0) splits = h->tune_attn_splits;
        splits = std::min(splits, h->max_splits);
        splits = std::min(splits, std::max(1, (S + 255) / 256));
        kps = ((S + splits - 1) / splits + 63) / 64 * 64;
        splits = (S + kps - 1) / kps;
    }
    a.n_splits = splits;
    a.keys_per_split = kps;
    const dim3 grid(q_tiles, c.n_q_heads, c.batch * splits);
    const int smem = 5 * 64 * c.head_dim * 2;
    switch (c.head_dim) {
        case 64:
            set_smem_attr_once(attention_kernel<64>, smem, h->device);
            launch_h(h, attention_kernel<64>, grid, 128, smem, a);
            break;
        case 128:
            set_smem_attr_once(attention_kernel<128>, smem, h->device);
            launch_h(h, attention_kernel<128>, grid, 128, smem, a);
            break;
        default:
            set_smem_attr_once(attention_kernel<256>, smem, h->device);
            launch_h(h, attention_kernel<256>, grid, 128, smem, a);
            break;
    }
    DGEN_TRY(check_launch(h));
    if (splits > 1) {
        const int rows = c.batch * c.n_q_heads * n_q;
        switch (c.head_dim) {
            case 64:
                launch_h(h, attention_combine_kernel<64>, (rows + 7) / 8, 256, 0, a);
                break;
            case 128:
                launch_h(h, attention_combine_kernel<128>, (rows + 7) / 8, 256, 0, a);
                break;
            default:
                launch_h(h, attention_combine_kernel<256>, (rows + 7) / 8, 256, 0, a);
                break;
        }
        DGEN_TRY(check_launch(h));
    }
    return DGEN_OK;
}

// The grouped expert GEMMs.  With a shared FFN (sh != null) its feature slices
// of width w are extra chunks (pseudo-experts E + j, appended by the routing
// permutation) of the same launch, reading the shared weights and the token
// rows in natural order.  With E4M3 experts (h->fp8) the operands are the
// quantized copies (weights made at create, token rows by the routing launch,
// activations by quant_rows_e4m3_kernel) and the epilogues apply their row scales.
struct SharedOperands {
    const CUtensorMap* w;    // shared gate-up / down weights (bf16 or E4M3)
    bf16* act_sh;
    float* y_sh;
    size_t rows_n;
};

// The gate-up and down launches' schedulers and epilogues, built once for the
// separate launches and for the fused one.
template <int KIND>
void gate_up_parts(dgen_handle* h, int l, const int4* chunks, const int* n_chunks, const SharedOperands* sh,
                   tc::GroupedSched& sc, EpiGateUp& ep) {
    const dgen_config& c = h->cfg;
    const int w = c.expert_width;
    sc = tc::GroupedSched{chunks, n_chunks, w / 64, 2 * w};
    for (int i = 0; i < 5; ++i) sc.tmBc[i] = KIND ? h->map_xperm8_c[i] : h->map_xperm_c[i];
    ep = EpiGateUp{h->act, w};
    if (KIND) {
        ep.w_scale = h->sgu + static_cast<size_t>(l) * c.n_experts * 2 * w;
        ep.x_scale = h->sxperm8;
        ep.w_scale_sh = h->ssgu + static_cast<size_t>(l) * 2 * c.shared_width;
        ep.x_scale_sh = h->sxn8;
    }
    if (sh) {
        sc.E = c.n_experts;
        sc.shared_a_stride = 2 * w;
        sc.tmA2 = *sh->w;
        for (int i = 0; i < 5; ++i) sc.tmB2c[i] = KIND ? h->map_xn8_c[i] : h->map_xn_c[i];
        ep.E = c.n_experts;
        ep.act_sh = sh->act_sh;
        ep.width_sh = c.shared_width;
    }
}

template <int KIND>
void down_parts(dgen_handle* h, int l, const int4* chunks, const int* n_chunks, const float* gate, float* y,
                const SharedOperands* sh, tc::GroupedSched& sc, EpiDown& ep) {
    const dgen_config& c = h->cfg;
    const int w = c.expert_width;
    sc = tc::GroupedSched{chunks, n_chunks, c.d_model / tc::BM, c.d_model};
    for (int i = 0; i < 5; ++i) sc.tmBc[i] = KIND ? h->map_act8_c[i] : h->map_act_c[i];
    ep = EpiDown{y, gate, c.d_model};
    if (KIND) {
        ep.w_scale = h->sd + static_cast<size_t>(l) * c.n_experts * c.d_model;
        ep.a_scale = h->sact8;
        ep.w_scale_sh = h->ssd + static_cast<size_t>(l) * c.d_model;
        ep.a_scale_sh = h->sactsh8;
    }
    if (sh) {
        sc.E = c.n_experts;
        sc.shared_k_off = KIND ? h->wpad : w;  // E4M3: each shared slice padded to whole 128-element k-blocks
        sc.tmA2 = *sh->w;
        for (int i = 0; i < 5; ++i) sc.tmB2c[i] = KIND ? h->map_actsh8_c[i] : h->map_actsh_c[i];
        ep.E = c.n_experts;
        ep.y_sh = sh->y_sh;
        ep.sh_stride = sh->rows_n * c.d_model;
    }
}

template <int BN, int KIND>
int grouped_gate_up(dgen_handle* h, int l, const int4* chunks, const int* n_chunks, int max_chunks,
                    const SharedOperands* sh) {
    const dgen_config& c = h->cfg;
    const int w = c.expert_width;
    tc::GroupedSched sc;
    EpiGateUp ep{nullptr, 0};
    gate_up_parts<KIND>(h, l, chunks, n_chunks, sh, sc, ep);
    sc.queue = h->tune_static_items ? nullptr : h->queue_l(l, 1);
    const int grid = std::min(h->num_sms, max_chunks * (w / 64));
    return launch_gemm<BN, 1, tc::GroupedSched, EpiGateUp, KIND>(h->stream, h->device, h->err,
                                                                 KIND ? h->maps[l].wgu8 : h->maps[l].wgu, sc.tmBc[0],
                                                                 sc, ep, c.d_model, grid, &h->launches);
}

template <int BN, int KIND>
int grouped_down(dgen_handle* h, int l, const int4* chunks, const int* n_chunks, int max_chunks, const float* gate,
                 float* y, const SharedOperands* sh) {
    const dgen_config& c = h->cfg;
    tc::GroupedSched sc;
    EpiDown ep{nullptr, nullptr, 0};
    down_parts<KIND>(h, l, chunks, n_chunks, gate, y, sh, sc, ep);
    sc.queue = h->tune_static_items ? nullptr : h->queue_l(l, 2);
    const int grid = std::min(h->num_sms, max_chunks * (c.d_model / tc::BM));
    return launch_gemm<BN, 1, tc::GroupedSched, EpiDown, KIND>(h->stream, h->device, h->err,
                                                               KIND ? h->maps[l].wd8 : h->maps[l].wd, sc.tmBc[0], sc,
                                                               ep, c.expert_width, grid, &h->launches);
}

// Both expert GEMMs in one persistent launch (bf16 operands): the grid is at
// most one CTA per SM, which the readiness waits of the down items rely on.
template <int BN>
int fused_experts(dgen_handle* h, int l, const int4* chunks, const int* n_chunks, int max_chunks, const float* gate,
                  float* y, const SharedOperands* sg, const SharedOperands* sd) {
    const dgen_config& c = h->cfg;
    tc::FusedExpertSched sc;
    EpiFusedExpert ep{EpiGateUp{nullptr, 0}, EpiDown{nullptr, nullptr, 0}, h->ready_l(l)};
    gate_up_parts<0>(h, l, chunks, n_chunks, sg, sc.gu, ep.gu);
    down_parts<0>(h, l, chunks, n_chunks, gate, y, sd, sc.dn, ep.dn);
    sc.tmA_gu = h->maps[l].wgu;
    sc.tmA_dn = h->maps[l].wd;
    sc.kb_gu = (c.d_model + tc::BK - 1) / tc::BK;
    sc.kb_dn = (c.expert_width + tc::BK - 1) / tc::BK;
    sc.ready = h->ready_l(l);
    sc.queue = h->tune_static_items ? nullptr : h->queue_l(l);
    const int items = max_chunks * (c.expert_width / 64 + c.d_model / tc::BM);
    const int grid = std::min(h->num_sms, items);
    return launch_gemm<BN, 1, tc::FusedExpertSched, EpiFusedExpert, 0>(h->stream, h->device, h->err,
                                                                       h->maps[l].wgu, sc.gu.tmBc[0], sc, ep,
                                                                       c.d_model, grid, &h->launches);
}

int dispatch_fused(dgen_handle* h, int bn, int l, const int4* chunks, const int* n_chunks, int max_chunks,
                   const float* gate, float* y, const SharedOperands* sg, const SharedOperands* sd) {
    switch (bn) {
        case 32: return fused_experts<32>(h, l, chunks, n_chunks, max_chunks, gate, y, sg, sd);
        case 64: return fused_experts<64>(h, l, chunks, n_chunks, max_chunks, gate, y, sg, sd);
        case 128: return fused_experts<128>(h, l, chunks, n_chunks, max_chunks, gate, y, sg, sd);
        default: return fused_experts<256>(h, l, chunks, n_chunks, max_chunks, gate, y, sg, sd);
    }
}

template <int KIND>
int dispatch_gate_up_k(dgen_handle* h, int bn, int l, const int4* chunks, const int* n_chunks, int max_chunks,
                       const SharedOperands* sh) {
    switch (bn) {
        case 32: return grouped_gate_up<32, KIND>(h, l, chunks, n_chunks, max_chunks, sh);
        case 64: return grouped_gate_up<64, KIND>(h, l, chunks, n_chunks, max_chunks, sh);
        case 128: return grouped_gate_up<128, KIND>(h, l, chunks, n_chunks, max_chunks, sh);
        default: return grouped_gate_up<256, KIND>(h, l, chunks, n_chunks, max_chunks, sh);
    }
}

template <int KIND>
int dispatch_down_k(dgen_handle* h, int bn, int l, const int4* chunks, const int* n_chunks, int max_chunks,
                    const float* gate, float* y, const SharedOperands* sh) {
    switch (bn) {
        case 32: return grouped_down<32, KIND>(h, l, chunks, n_chunks, max_chunks, gate, y, sh);
        case 64: return grouped_down<64, KIND>(h, l, chunks, n_chunks, max_chunks, gate, y, sh);
        case 128: return grouped_down<128, KIND>(h, l, chunks, n_chunks, max_chunks, gate, y, sh);
        default: return grouped_down<256, KIND>(h, l, chunks, n_chunks, max_chunks, gate, y, sh);
    }
}

int dispatch_gate_up(dgen_handle* h, int bn, int l, const int4* chunks, const int* n_chunks, int max_chunks,
                     const SharedOperands* sh) {
    return h->fp8 ? dispatch_gate_up_k<1>(h, bn, l, chunks, n_chunks, max_chunks, sh)
                  : dispatch_gate_up_k<0>(h, bn, l, chunks, n_chunks, max_chunks, sh);
}

int dispatch_down(dgen_handle* h, int bn, int l, const int4* chunks, const int* n_chunks, int max_chunks,
                  const float* gate, float* y, const SharedOperands* sh) {
    return h->fp8 ? dispatch_down_k<1>(h, bn, l, chunks, n_chunks, max_chunks, gate, y, sh)
                  : dispatch_down_k<0>(h, bn, l, chunks, n_chunks, max_chunks, gate, y, sh);
}

// Number of K splits for a GEMM with `tiles` output tiles and num_kb k-blocks:
// enough splits to occupy about `target` CTAs, every split non-empty.
int k_splits_for(int tiles, int num_kb, int target) {
    const int want = std::max(1, std::min(num_kb, target / std::max(1, tiles)));
    const int per = (num_kb + want - 1) / want;
    return (num_kb + per - 1) / per;
}

// Grid of the routing kernel for `rows` token rows: (CTAs, tokens per CTA).
void route_grid(const dgen_handle* h, int rows, int& grid, int& tb) {
    grid = std::max(1, std::min({h->num_sms, kRouteMaxGrid, (rows + 1) / 2}));
    tb = (rows + grid - 1) / grid;
    grid = (rows + tb - 1) / tb;
}

// Router logits (GEMM split over K, fp32 partials), then one routing launch:
// top-k + gates, the expert permutation and chunk list, the gather of the
// normed rows into expert order (moe_route_kernel).
int route(dgen_handle* h, int l, int rows, bool capture, const int32_t* forced, int chunk) {
    const dgen_config& c = h->cfg;
    const int E = c.n_experts;
    const int m_tiles = (rows + tc::BM - 1) / tc::BM;
    const int num_kb = (c.d_model + tc::BK - 1) / tc::BK;
    const int target = h->tune_router_splits > 0 ? h->tune_router_splits * m_tiles : 16;
    int ks = std::min({k_splits_for(m_tiles, num_kb, target), h->router_max_splits(rows), kRouteMaxParts});
    ks = (num_kb + (num_kb + ks - 1) / ks - 1) / ((num_kb + ks - 1) / ks);  // every split non-empty
    tc::DenseSched sc{m_tiles, 1, ks, 1};
    EpiStoreF32 ep{h->rlogits, rows, E, E, static_cast<size_t>(rows) * E};
    const CUtensorMap& wr = h->maps[l].wr;
    const int grid = std::min(h->num_sms, m_tiles * ks);
    int rc;
    switch (h->bn_router) {
        case 16: rc = launch_gemm<16, 1>(h->stream, h->device, h->err, h->map_xn_a, wr, sc, ep, c.d_model, grid, &h->launches); break;
        case 32: rc = launch_gemm<32, 1>(h->stream, h->device, h->err, h->map_xn_a, wr, sc, ep, c.d_model, grid, &h->launches); break;
        case 64: rc = launch_gemm<64, 1>(h->stream, h->device, h->err, h->map_xn_a, wr, sc, ep, c.d_model, grid, &h->launches); break;
        case 128: rc = launch_gemm<128, 1>(h->stream, h->device, h->err, h->map_xn_a, wr, sc, ep, c.d_model, grid, &h->launches); break;
        default: rc = launch_gemm<256, 1>(h->stream, h->device, h->err, h->map_xn_a, wr, sc, ep, c.d_model, grid, &h->launches); break;
    }
    DGEN_TRY(rc);
    RouteArgs a{};
    a.parts = h->rlogits;
    a.n_parts = ks;
    a.rows = rows;
    a.E = E;
    a.k = c.top_k;
    int rgrid = 1;
    route_grid(h, rows, rgrid, a.TB);
    a.topk_id = h->topk_id;
    a.topk_gate = h->topk_gate;
    a.logits_out = (capture && h->cap_logits) ? h->cap_logits + static_cast<size_t>(l) * rows * E : nullptr;
    a.forced = forced;
    a.chunk = chunk;
    a.n_shared = h->n_shared_parts;
    a.perm_tok = h->perm_tok;
    a.perm_gate = h->perm_gate;
    a.inv = h->inv;
    a.chunks = h->chunks;
    a.n_chunks = h->n_chunks;
    a.n_touched = h->touched + l;
    a.xn = h->xn;
    a.xperm = h->xperm;
    a.xperm8 = h->fp8 ? h->xperm8 : nullptr;
    a.sxperm8 = h->sxperm8;
    a.xn8 = h->xn8;
    a.sxn8 = h->sxn8;
    a.d = c.d_model;
    a.tot = h->route_tot(l);
    a.barrier = h->barriers + l;
    a.barrier_extra = h->route_barrier_extra;
    a.err = h->err;
    const size_t smem = route_smem_bytes(E, a.TB, a.k);
    // routed chunks: automatic = largest expert first where the expert GEMMs run as
    // two launches (E4M3 experts), expert id order for the one persistent launch
    const bool by_size = h->tune_chunk_order ? h->tune_chunk_order == 2 : (h->fp8 || h->tune_separate_experts);
    if (by_size) {
        set_smem_attr_once(moe_route_kernel<true>, static_cast<int>(smem), h->device);
        launch_h(h, moe_route_kernel<true>, rgrid, kRouteThreads, smem, a);
    } else {
        set_smem_attr_once(moe_route_kernel<false>, static_cast<int>(smem), h->device);
        launch_h(h, moe_route_kernel<false>, rgrid, kRouteThreads, smem, a);
    }
    return check_launch(h);
}

// One transformer layer over `rows` rows (B sequences x n_q rows), queries at
// positions pos0.., keys 0..S-1 of the cache.  On entry h->xn holds the layer's
// attention-normed input (written by the previous kernel); the layer's last
// kernel writes the next normed input with gain next_norm (the next layer's
// attention norm, or the final norm), unless next_norm is null.  Prompt pass:
// causal attention, and the last layer stops after writing its K/V.
int run_layer(dgen_handle* h, int l, int rows, int n_q, int pos0, int S, bool prompt, const void* next_norm) {
    const dgen_config& c = h->cfg;
    const dgen_layer_weights& w = h->layers[l];
    const LayerMaps& m = h->maps[l];
    const int d = c.d_model;

    {
        Timed t(h, DGEN_K_QKV);
        const int heads = c.n_q_heads + 2 * c.n_kv_heads, width = heads * c.head_dim;
        const int m_tiles = (rows + tc::BM - 1) / tc::BM, tiles = m_tiles * heads;
        const int num_kb = (d + tc::BK - 1) / tc::BK;
        // K split + a second kernel that sums the partials, rotates and scatters:
        // measured slower than the fused RoPE epilogue at every workload here, so
        // only on request (DGEN_TUNE_QKV_SPLITS)
        int qs = h->tune_qkv_splits > 0 ? h->tune_qkv_splits : 1;
        (void)num_kb;
        qs = std::min<int>(qs, static_cast<int>(h->qkv_parts_rows / rows));
        const int grid_tiles = tiles * std::max(qs, 1);
        const int grid = std::min(h->num_sms, grid_tiles);
        if (qs <= 1 && c.head_dim == 256 && h->tune_pairs == 2) {
            // CTA pairs over 256 rows x 128 features: CTA 0 loads 64 features, CTA 1
            // their rotate-half partners (RopePairSched), RoPE in the epilogue
            tc2::RopePairSched sc;
            sc.m_tiles = (rows + 255) / 256;
            sc.n_tiles = heads * 2;
            sc.k_splits = 1;
            sc.b_static = 1;
            sc.pair_off = c.head_dim / 2;
            EpiQKVPair ep{h->q, h->kc_l(l), h->vc_l(l), h->rope, rows, n_q, pos0, c.n_q_heads, c.n_kv_heads,
                          c.head_dim, h->S_max};
            DGEN_TRY(launch_gemm_pair<128>(h->stream, h->device, h->err, h->map_xn_a, m.wqkv_pair, sc, ep, d,
                                           std::min(h->num_sms / 2, sc.m_tiles * sc.n_tiles), &h->launches));
        } else if (qs <= 1 && c.head_dim == 256) {
            // 128-wide tiles holding RoPE pairs (PairSched): twice the CTAs of whole-head tiles
            tc::PairSched sc;
            sc.m_tiles = m_tiles;
            sc.n_tiles = heads * 2;
            sc.k_splits = 1;
            sc.b_static = 1;
            sc.pair_off = c.head_dim / 2;
            EpiQKVPair ep{h->q, h->kc_l(l), h->vc_l(l), h->rope, rows, n_q, pos0, c.n_q_heads, c.n_kv_heads,
                          c.head_dim, h->S_max};
            DGEN_TRY(launch_gemm<128, 1>(h->stream, h->device, h->err, h->map_xn_a, m.wqkv_pair, sc, ep, d,
                                         std::min(h->num_sms, m_tiles * heads * 2), &h->launches));
        } else if (qs <= 1) {
            tc::DenseSched sc{m_tiles, heads, 1, 1};
            EpiQKV ep{h->q, h->kc_l(l), h->vc_l(l), h->rope, rows, n_q, pos0, c.n_q_heads, c.n_kv_heads,
                      c.head_dim, h->S_max};
            if (c.head_dim == 256)
                DGEN_TRY(launch_gemm<256, 1>(h->stream, h->device, h->err, h->map_xn_a, m.wqkv, sc, ep, d, grid, &h->launches));
            else if (c.head_dim == 128)
                DGEN_TRY(launch_gemm<128, 1>(h->stream, h->device, h->err, h->map_xn_a, m.wqkv, sc, ep, d, grid, &h->launches));
            else
                DGEN_TRY(launch_gemm<64, 1>(h->stream, h->device, h->err, h->map_xn_a, m.wqkv, sc, ep, d, grid, &h->launches));
        } else {
            tc::DenseSched sc{m_tiles, heads, qs, 1};
            const size_t stride = static_cast<size_t>(rows) * width;
            EpiStoreF32 ep{h->qkv_parts, rows, width, width, stride};
            if (c.head_dim == 256)
                DGEN_TRY(launch_gemm<256, 1>(h->stream, h->device, h->err, h->map_xn_a, m.wqkv, sc, ep, d, grid, &h->launches));
            else if (c.head_dim == 128)
                DGEN_TRY(launch_gemm<128, 1>(h->stream, h->device, h->err, h->map_xn_a, m.wqkv, sc, ep, d, grid, &h->launches));
            else
                DGEN_TRY(launch_gemm<64, 1>(h->stream, h->device, h->err, h->map_xn_a, m.wqkv, sc, ep, d, grid, &h->launches));
            launch_h(h, rope_scatter_kernel, dim3(rows, heads), dim3(c.head_dim / 2), 0,
                     static_cast<const float*>(h->qkv_parts), qs, stride, rows, n_q, pos0, c.n_q_heads, c.n_kv_heads,
                     c.head_dim, h->S_max, static_cast<const float2*>(h->rope), h->q, h->kc_l(l), h->vc_l(l));
            DGEN_TRY(check_launch(h));
        }
    }
    if (prompt && l == c.n_layers - 1) return DGEN_OK;
    {
        Timed t(h, DGEN_K_ATTENTION);
        DGEN_TRY(attention(h, l, n_q, S, pos0, prompt));
    }
    int os = 1;
    {
        // O projection over 128-wide column tiles, split over K into fp32 partials
        // that the next kernel adds to the residual (in split order) before the norm
        Timed t(h, DGEN_K_OPROJ);
        const int m_tiles = (rows + tc::BM - 1) / tc::BM, n_tiles = d / tc::BM, tiles = m_tiles * n_tiles;
        const int K = c.n_q_heads * c.head_dim, num_kb = (K + tc::BK - 1) / tc::BK;
        os = k_splits_for(tiles, num_kb, h->num_sms);
        os = std::max(1, std::min<int>({os, static_cast<int>(h->oparts_rows / rows), kMaxParts}));
        os = (num_kb + (num_kb + os - 1) / os - 1) / ((num_kb + os - 1) / os);  // every split non-empty
        EpiStoreF32 ep{h->oparts, rows, d, d, static_cast<size_t>(rows) * d};
        if (h->tune_pairs == 2 && d % 256 == 0) {
            // CTA pairs over 256 rows x 256 columns, K split so that the pairs fill the SMs
            const int pm = (rows + 255) / 256, pn = d / 256, ptiles = pm * pn;
            int ps = k_splits_for(ptiles, num_kb, h->num_sms / 2);
            ps = std::max(1, std::min<int>({ps, static_cast<int>(h->oparts_rows / rows), kMaxParts}));
            ps = (num_kb + (num_kb + ps - 1) / ps - 1) / ((num_kb + ps - 1) / ps);  // every split non-empty
            os = ps;
            tc2::DensePairSched sc;
            sc.m_tiles = pm;
            sc.n_tiles = pn;
            sc.k_splits = ps;
            sc.b_static = 1;
            DGEN_TRY(launch_gemm_pair<256>(h->stream, h->device, h->err, h->map_attn_a, m.wo, sc, ep, K,
                                           std::min(h->num_sms / 2, ptiles * ps), &h->launches));
        } else {
            tc::DenseSched sc{m_tiles, n_tiles, os, 1};
            DGEN_TRY(launch_gemm<128, 1>(h->stream, h->device, h->err, h->map_attn_a, m.wo, sc, ep, K,
                                         std::min(h->num_sms, tiles * os), &h->launches));
        }
    }
    {
        Timed t(h, DGEN_K_OTHER);
        launch_h(h, residual_norm_kernel, rows, row_threads(d), 0, h->h, static_cast<const float*>(h->oparts), os,
                 static_cast<size_t>(rows) * d, rows, d, static_cast<const uint16_t*>(w.ffn_norm), h->xn, c.rms_eps);
        DGEN_TRY(check_launch(h));
    }
    const int nk = rows * c.top_k;
    const int chunk = h->tune_chunk > 0 ? h->tune_chunk : pick_chunk(static_cast<double>(nk) / c.n_experts);
    const int n_sh = h->n_shared_parts;
    const int max_chunks = std::min(h->max_chunks, c.n_experts + (nk + chunk - 1) / chunk +
                                                       n_sh * ((rows + chunk - 1) / chunk));
    {
        Timed t(h, DGEN_K_ROUTER);
        const int32_t* forced = prompt ? h->force_prompt : h->force_canvas;
        DGEN_TRY(route(h, l, rows, !prompt, forced ? forced + static_cast<size_t>(l) * nk : nullptr, chunk));
        if (!prompt && h->cap_ids &&
            cudaMemcpyAsync(h->cap_ids + static_cast<size_t>(l) * nk, h->topk_id, static_cast<size_t>(nk) * sizeof(int),
                            cudaMemcpyDeviceToDevice, h->stream) != cudaSuccess)
            return DGEN_ECUDA;
    }
    const size_t down_stride = static_cast<size_t>(nk) * d;
    SharedOperands sg{h->fp8 ? &m.wsgu8 : &m.wsgu, h->act_sh, h->y_sh, static_cast<size_t>(rows)};
    SharedOperands sd{h->fp8 ? &m.wsd8 : &m.wsd, h->act_sh, h->y_sh, static_cast<size_t>(rows)};
    if (!h->fp8 && !h->tune_separate_experts) {  // both expert GEMMs in one persistent launch
        Timed t(h, DGEN_K_EXPERT_GATE_UP);
        DGEN_TRY(dispatch_fused(h, chunk, l, h->chunks, h->n_chunks, max_chunks, h->perm_gate, h->yperm,
                                n_sh ? &sg : nullptr, n_sh ? &sd : nullptr));
    } else {
    {
        Timed t(h, DGEN_K_EXPERT_GATE_UP);
        DGEN_TRY(dispatch_gate_up(h, chunk, l, h->chunks, h->n_chunks, max_chunks, n_sh ? &sg : nullptr));
        if (h->fp8) {  // the gated activations -> E4M3 rows for the down GEMM
            const int w = c.expert_width;
            launch_h(h, quant_rows_e4m3_kernel, (nk + 7) / 8, 256, 0, static_cast<const bf16*>(h->act),
                     static_cast<size_t>(w), nk, w, h->act8, static_cast<size_t>(w), w, w, h->sact8);
            DGEN_TRY(check_launch(h));
            if (n_sh) {
                launch_h(h, quant_rows_e4m3_kernel, (rows + 7) / 8, 256, 0, static_cast<const bf16*>(h->act_sh),
                         static_cast<size_t>(c.shared_width), rows, c.shared_width, h->actsh8,
                         static_cast<size_t>(n_sh) * h->wpad, w, h->wpad, h->sactsh8);
                DGEN_TRY(check_launch(h));
            }
        }
    }
    {
        Timed t(h, DGEN_K_EXPERT_DOWN);
        DGEN_TRY(dispatch_down(h, chunk, l, h->chunks, h->n_chunks, max_chunks, h->perm_gate, h->yperm,
                               n_sh ? &sd : nullptr));
    }
    }
    Timed t(h, DGEN_K_OTHER);
    launch_h(h, moe_combine_norm_kernel, rows, row_threads(d), 0, h->h, static_cast<const float*>(h->yperm), down_stride, 1,
             static_cast<const int*>(h->inv), static_cast<const float*>(h->y_sh), n_sh, rows, c.top_k, d,
             static_cast<const uint16_t*>(next_norm), h->xn, c.rms_eps);
    return check_launch(h);
}

// log2(e) / tau_s into slot `slot` of the handle's 1/tau words (0: the step's LM-head
// statistics and the fixed-count sampler; 1: the entropy-bounded sampler on given logits).
int set_tau(dgen_handle* h, int s, int T, int slot = 0) {
    const double t = 1.0 - static_cast<double>(s) / T;
    const double tau = h->cfg.tau_min + (static_cast<double>(h->cfg.tau_max) - h->cfg.tau_min) * t;
    launch_h(h, set_inv_tau_kernel, 1, 1, 0, h->inv_tau + slot, static_cast<float>(1.4426950408889634 / tau));
    return check_launch(h);
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Philox position of canvas index 0 for the current block: canvases appended to
// the cache since the prompt x C, so every block of a sequence draws fresh words.
uint32_t pos_offset(const dgen_handle* h) { return static_cast<uint32_t>(h->blocks_done) * h->cfg.canvas; }

int validate(const dgen_config* c, const dgen_weights* w) {
    if (!c || !w || !w->layers) return DGEN_EINVAL;
    if (c->n_layers < 1 || c->d_model < 128 || c->d_model % 128 || c->d_model > 4096) return DGEN_EINVAL;
    if (c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256) return DGEN_EINVAL;
    if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads) return DGEN_EINVAL;
    if (c->n_experts < 1 || c->n_experts > 256 || c->top_k < 1 || c->top_k > kMaxTopKRouting ||
        c->top_k > c->n_experts)
        return DGEN_EINVAL;
    if (c->expert_width < 64 || c->expert_width % 64 || c->shared_width < 0 || c->shared_width % 64)
        return DGEN_EINVAL;
    // the shared FFN runs as ceil(ws / w) pseudo-experts; the combine sums at most kMaxParts of them
    if ((c->shared_width + c->expert_width - 1) / c->expert_width > kMaxParts) return DGEN_EINVAL;
    if (c->vocab < 256 || c->vocab % 256) return DGEN_EINVAL;
    if (c->batch < 1 || c->prompt_max < 1 || c->canvas < 1 || c->canvas > 1024 || c->commit_per_step < 0)
        return DGEN_EINVAL;
    if (!(c->tau_max > 0.f) || !(c->tau_min > 0.f) || !(c->rms_eps >= 0.f) || !(c->rope_base > 0.f))
        return DGEN_EINVAL;
    if (c->expert_fp8 != 0 && c->expert_fp8 != 1) return DGEN_EINVAL;
    if (!aligned16(w->embed) || !aligned16(w->final_norm)) return DGEN_EINVAL;
    for (int l = 0; l < c->n_layers; ++l) {
        const dgen_layer_weights& L = w->layers[l];
        if (!aligned16(L.attn_norm) || !aligned16(L.w_qkv) || !aligned16(L.w_o) || !aligned16(L.ffn_norm) ||
            !aligned16(L.w_router) || !aligned16(L.w_gate_up) || !aligned16(L.w_down))
            return DGEN_EINVAL;
        if (c->shared_width > 0 && (!aligned16(L.w_shared_gate_up) || !aligned16(L.w_shared_down)))
            return DGEN_EINVAL;
    }
    if (c->self_cond_width < 0 || c->self_cond_width % 64) return DGEN_EINVAL;
    if (c->self_cond_width > 0 &&
        (!aligned16(w->sc_norm) || !aligned16(w->w_sc_gate_up) || !aligned16(w->w_sc_down)))
        return DGEN_EINVAL;
    return DGEN_OK;
}

// K splits of the p0_hat E GEMM (tiles output tiles, num_kb k-blocks over the
// vocabulary): the persistent grid's critical path in k-blocks, ceil(tiles s /
// SMs) x ceil(num_kb / s), plus the partials' extra traffic (written and read
// once per split) in units of one k-block's operand bytes on every SM.  Every
// split non-empty.
int sc_pe_splits(int tiles, int num_kb, int sms, double part_bytes, double kb_bytes) {
    int best = 1;
    double best_cost = 1e300;
    for (int s = 1; s <= kMaxScSplits && s <= num_kb; ++s) {
        const double waves = static_cast<double>((tiles * s + sms - 1) / sms);
        const double cost = waves * ((num_kb + s - 1) / s) + s * 2.0 * part_bytes / (sms * kb_bytes);
        if (cost < best_cost) {
            best = s;
            best_cost = cost;
        }
    }
    const int per = (num_kb + best - 1) / best;
    return (num_kb + per - 1) / per;
}

void free_all(dgen_handle* h) {
    for (void* p : h->allocs) cudaFree(p);
    h->allocs.clear();
    if (h->host_flags) cudaFreeHost(h->host_flags);
    h->host_flags = nullptr;
}

// Self-conditioning (hyper.ai digest, Method, eqs. 3-4): from the pass's logits
// and the LM head's row statistics, z = FFW(p0_hat E) for every canvas row:
// p0_hat (bf16), u = p0_hat E as a K-split GEMM over the vocabulary with the
// embedding read MN-major, RMSNorm(u), the gated-GELU gate-up GEMM, the down
// GEMM into z's K-split partials (summed by the next pass's embedding kernel).
int self_cond(dgen_handle* h, const float* logits) {
    const dgen_config& c = h->cfg;
    const int rows = h->rows_c, d = c.d_model, w = c.self_cond_width;
    const int m_tiles = (rows + tc::BM - 1) / tc::BM;
    Timed t(h, DGEN_K_SELF_COND);
    launch_h(h, sc_probs_kernel, rows * h->sc_slices, 256, 0, logits, static_cast<const float*>(h->pmax),
             static_cast<const float*>(h->psum), c.vocab / 256, c.vocab, static_cast<const float*>(h->inv_tau),
             h->sc_p, h->sc_slices);
    DGEN_TRY(check_launch(h));
    const size_t part = static_cast<size_t>(rows) * d;
    EpiStoreF32 eu{h->sc_u, rows, d, d, part};
    int grid;
    if (h->sc_pairs && h->tune_pairs != 1) {  // CTA pairs over 256 rows x 256 columns of d
        tc2::DensePairMNSched pe;
        pe.m_tiles = (rows + 255) / 256;
        pe.n_tiles = d / 256;
        pe.k_splits = h->sc_ks;
        pe.b_static = 1;
        DGEN_TRY(launch_gemm_pair<256>(h->stream, h->device, h->err, h->map_sc_p, h->map_embed_mn, pe, eu, c.vocab,
                                       std::min(h->num_sms / 2, pe.m_tiles * pe.n_tiles * pe.k_splits),
                                       &h->launches));
    } else {
        tc::DenseMNSched pe;
        pe.m_tiles = m_tiles;
        pe.n_tiles = d / h->sc_bn_pe;
        pe.k_splits = h->sc_ks;
        pe.b_static = 1;
        grid = std::min(h->num_sms, pe.m_tiles * pe.n_tiles * pe.k_splits);
        DGEN_TRY(h->sc_bn_pe == 256 ? launch_gemm<256, 1>(h->stream, h->device, h->err, h->map_sc_p, h->map_embed_mn,
                                                          pe, eu, c.vocab, grid, &h->launches)
                                    : launch_gemm<128, 1>(h->stream, h->device, h->err, h->map_sc_p, h->map_embed_mn,
                                                          pe, eu, c.vocab, grid, &h->launches));
    }
    launch_h(h, sc_norm_kernel, rows, 128, 0, static_cast<const float*>(h->sc_u), h->sc_ks, part, rows, d,
             h->sc_norm, h->sc_n, c.rms_eps);
    DGEN_TRY(check_launch(h));
    tc::DenseSched gu{m_tiles, 2 * w / h->sc_bn_gu, 1, 1};
    EpiGateUpDense eg{h->sc_act, w, rows};
    grid = std::min(h->num_sms, gu.m_tiles * gu.n_tiles);
    DGEN_TRY(h->sc_bn_gu == 128 ? launch_gemm<128, 1>(h->stream, h->device, h->err, h->map_sc_n, h->map_sc_wgu, gu,
                                                      eg, d, grid, &h->launches)
                                : launch_gemm<64, 1>(h->stream, h->device, h->err, h->map_sc_n, h->map_sc_wgu, gu, eg,
                                                     d, grid, &h->launches));
    tc::DenseSched dn{m_tiles, d / 128, h->sc_kz, 1};
    EpiStoreF32 ez{h->sc_z, rows, d, d, part};
    grid = std::min(h->num_sms, dn.m_tiles * dn.n_tiles * dn.k_splits);
    return launch_gemm<128, 1>(h->stream, h->device, h->err, h->map_sc_act, h->map_sc_wd, dn, ez, w, grid,
                               &h->launches);
}

// Clears the self-conditioning state (z = 0 at the first step of a block).
int sc_clear(dgen_handle* h) {
    if (!h->sc) return DGEN_OK;
    return cudaMemsetAsync(h->sc_z, 0, h->sc_z_bytes(), h->stream) == cudaSuccess ? DGEN_OK : DGEN_ECUDA;
}

// The decoder pass after set_tau: embedding, L layers, final norm + LM head
// (+ the self-conditioning state for the next pass).
int step_body(dgen_handle* h, float* logits) {
    const dgen_config& c = h->cfg;
    const int rows = h->rows_c, P = h->P;
    {
        Timed t(h, DGEN_K_OTHER);
        DGEN_TRY(embed(h, h->tok, rows, h->sc ? h->sc_z : nullptr));
    }
    for (int l = 0; l < c.n_layers; ++l) {
        DGEN_TRY(run_layer(h, l, rows, c.canvas, P, P + c.canvas, false, next_norm_of(h, l)));
        if (h->cap_h &&
            cudaMemcpyAsync(h->cap_h + static_cast<size_t>(l) * rows * c.d_model, h->h,
                            static_cast<size_t>(rows) * c.d_model * sizeof(float), cudaMemcpyDeviceToDevice,
                            h->stream) != cudaSuccess)
            return DGEN_ECUDA;
    }
    float* lg = logits ? logits : (h->sc ? h->sc_logits : nullptr);
    {
        Timed t(h, DGEN_K_LM_HEAD);  // h->xn holds the final-normed state (fused into the last combine)
        EpiLMHead ep{h->pmax, h->psum, h->pent, h->parg, lg, h->inv_tau, rows, c.vocab, c.vocab / 256};
        if (h->tune_pairs != 1) {  // CTA pairs over 256 rows x 256 vocabulary rows
            tc2::DensePairSched sc;
            sc.m_tiles = (rows + 255) / 256;
            sc.n_tiles = c.vocab / 256;
            sc.k_splits = 1;
            sc.b_static = 1;
            DGEN_TRY(launch_gemm_pair<256>(h->stream, h->device, h->err, h->map_xn_a, h->map_embed_b128, sc, ep,
                                           c.d_model, std::min(h->num_sms / 2, sc.m_tiles * sc.n_tiles),
                                           &h->launches));
        } else {
            tc::DenseSched sc{(rows + tc::BM - 1) / tc::BM, c.vocab / 256, 1, 1};
            const int grid = std::min(h->num_sms, sc.m_tiles * sc.n_tiles);
            DGEN_TRY(launch_gemm<256, 1>(h->stream, h->device, h->err, h->map_xn_a, h->map_embed_b, sc, ep,
                                         c.d_model, grid, &h->launches));
        }
    }
    return h->sc ? self_cond(h, lg) : DGEN_OK;
}

void release_graph(dgen_handle* h) {
    if (h->graph) cudaGraphExecDestroy(h->graph);
    h->graph = nullptr;
    for (const auto& p : h->graph_pairs) {
        h->ev_pool.push_back(p.a);
        h->ev_pool.push_back(p.b);
    }
    h->graph_pairs.clear();
}

// Captures step_body into a CUDA graph on the handle's stream.  Leaves
// h->graph null (and disables graphs) if the stream cannot be captured.
int capture_step(dgen_handle* h) {
    if (cudaStreamBeginCapture(h->stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        cudaGetLastError();
        h->use_graph = false;
        return DGEN_OK;
    }
    const size_t timed0 = h->timed.size();
    const int64_t launches0 = h->launches;
    const int rc = step_body(h, nullptr);
    cudaGraph_t g = nullptr;
    const cudaError_t e = cudaStreamEndCapture(h->stream, &g);
    h->graph_launches = h->launches - launches0;
    h->launches = launches0;
    h->graph_pairs.assign(h->timed.begin() + timed0, h->timed.end());
    h->timed.resize(timed0);
    if (rc != DGEN_OK || e != cudaSuccess || !g) {
        if (g) cudaGraphDestroy(g);
        release_graph(h);
        return rc != DGEN_OK ? rc : DGEN_ECUDA;
    }
    const cudaError_t ei = cudaGraphInstantiate(&h->graph, g, 0);
    cudaGraphDestroy(g);
    if (ei != cudaSuccess) {
        h->graph = nullptr;
        release_graph(h);
        return DGEN_ECUDA;
    }
    h->graph_P = h->P;
    h->graph_mask = h->timing_mask;
    h->graph_force = h->force_canvas;
    return DGEN_OK;
}

}  // namespace

// ================================================================== C ABI

extern "C" {

const char* dgen_status_str(int status) {
    switch (status) {
        case DGEN_OK: return "ok";
        case DGEN_EINVAL: return "invalid argument or unsupported shape";
        case DGEN_ENOMEM: return "device allocation failed";
        case DGEN_ECAP: return "prompt longer than prompt_max";
        case DGEN_ECUDA: return "CUDA error";
        case DGEN_EDEVICE: return "a device-side bounded wait ran out";
        case DGEN_ESTATE: return "call out of order";
        case DGEN_ESCRATCH: return "sizes exceed the fixed scratch of the allocation-free entry point";
        default: return "unknown status";
    }
}

int dgen_create(const dgen_config* cfg, const dgen_weights* weights, void* stream, dgen_handle** out) {
    if (!out) return DGEN_EINVAL;
    *out = nullptr;
    DGEN_TRY(validate(cfg, weights));
    if (!load_encode()) return DGEN_ECUDA;
    dgen_handle* h = new dgen_handle();
    const dgen_config& c = *cfg;
    h->cfg = c;
    h->embed = static_cast<const uint16_t*>(weights->embed);
    h->final_norm = static_cast<const uint16_t*>(weights->final_norm);
    h->layers.assign(weights->layers, weights->layers + c.n_layers);
    h->stream = static_cast<cudaStream_t>(stream);
    if (cudaGetDevice(&h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
        delete h;
        return DGEN_ECUDA;
    }
    const int B = c.batch, C = c.canvas, d = c.d_model, k = c.top_k, hd = c.head_dim;
    h->S_max = c.prompt_max + C;
    h->rows_c = B * C;
    h->rows_max = std::max(B * C, B * c.prompt_max);
    {
        int rg = 1, tb = 1;
        route_grid(h, h->rows_max, rg, tb);
        if (tb > kRouteMaxTB || tb * k > kRouteMaxSlots) {  // too many rows for one routing launch
            delete h;
            return DGEN_EINVAL;
        }
    }
    h->bn_router = 16;
    while (h->bn_router < c.n_experts) h->bn_router *= 2;
    h->kv_layer = static_cast<size_t>(B) * c.n_kv_heads * h->S_max * hd;
    h->kv_P.assign(c.n_layers, -1);
    const size_t R = h->rows_max, RK = R * k;
    h->rlogits_rows = std::max<size_t>(R, 64 * tc::BM);
    h->qkv_parts_rows = 4 * static_cast<size_t>(B) * C;
    h->oparts_rows = std::max<size_t>(R, static_cast<size_t>(h->num_sms) * tc::BM);
    h->n_shared_parts = (c.shared_width + c.expert_width - 1) / c.expert_width;  // <= kMaxParts (validate)
    h->max_chunks = c.n_experts + static_cast<int>((RK + 31) / 32) + 1 +
                    h->n_shared_parts * static_cast<int>((R + 31) / 32);
    const int n_vt = c.vocab / 256;

    bool ok = h->alloc(&h->tok, static_cast<size_t>(B) * C) && h->alloc(&h->committed, static_cast<size_t>(B) * C) &&
              h->alloc(&h->kc, h->kv_layer * c.n_layers) && h->alloc(&h->vc, h->kv_layer * c.n_layers) &&
              h->alloc(&h->h, R * d) && h->alloc(&h->xn, R * d) &&
              h->alloc(&h->q, static_cast<size_t>(B) * c.n_q_heads * std::max(C, c.prompt_max) * hd) &&
              h->alloc(&h->attn, R * c.n_q_heads * hd) &&
              h->alloc(&h->part_o, static_cast<size_t>(h->max_splits) * B * c.n_q_heads * C * hd) &&
              h->alloc(&h->part_lse, static_cast<size_t>(h->max_splits) * B * c.n_q_heads * C) &&
              h->alloc(&h->rlogits, h->rlogits_rows * c.n_experts) &&
              h->alloc(&h->qkv_parts, h->qkv_parts_rows * (c.n_q_heads + 2 * c.n_kv_heads) * hd) &&
              h->alloc(&h->oparts, h->oparts_rows * d) && h->alloc(&h->topk_id, RK) &&
              h->alloc(&h->topk_gate, RK) && h->alloc(&h->perm_tok, RK) &&
              h->alloc(&h->perm_gate, RK) && h->alloc(&h->inv, RK) && h->alloc(&h->chunks, h->max_chunks) &&
              h->alloc(&h->n_chunks, 1) && h->alloc(&h->touched, c.n_layers) && h->alloc(&h->xperm, RK * d) &&
              h->alloc(&h->barriers, static_cast<size_t>(h->route_words())) &&
              h->alloc(&h->act, RK * c.expert_width) && h->alloc(&h->yperm, std::max<size_t>(RK, 2 * static_cast<size_t>(B) * C * k) * d) &&
              h->alloc(&h->act_sh, R * std::max(c.shared_width, 64)) &&
              h->alloc(&h->y_sh, c.shared_width > 0 ? h->n_shared_parts * R * d : 1) &&
              h->alloc(&h->pmax, static_cast<size_t>(B) * C * n_vt) &&
              h->alloc(&h->psum, static_cast<size_t>(B) * C * n_vt) &&
              h->alloc(&h->pent, static_cast<size_t>(B) * C * n_vt) && h->alloc(&h->eb_done, B) &&
              h->alloc(&h->parg, static_cast<size_t>(B) * C * n_vt) && h->alloc(&h->conf, static_cast<size_t>(B) * C) &&
              h->alloc(&h->argmax, static_cast<size_t>(B) * C) &&
              h->alloc(&h->eb_prev_argmax, static_cast<size_t>(B) * C) &&
              h->alloc(&h->rope, static_cast<size_t>(h->S_max) * (hd / 2)) && h->alloc(&h->inv_tau, 2) &&
              h->alloc(&h->err, 1) && h->alloc(&h->prompt_buf, static_cast<size_t>(B) * c.prompt_max);
    h->fp8 = c.expert_fp8 != 0;
    if (ok && h->fp8) {
        const size_t L = c.n_layers, E = c.n_experts, w = c.expert_width, ws = c.shared_width;
        const size_t nsh = h->n_shared_parts;
        h->wpad = (c.expert_width + 127) / 128 * 128;
        ok = h->alloc(&h->wgu8, L * E * 2 * w * d) && h->alloc(&h->sgu, L * E * 2 * w) &&
             h->alloc(&h->wd8, L * E * d * w) && h->alloc(&h->sd, L * E * d) &&
             h->alloc(&h->wsgu8, std::max<size_t>(1, L * 2 * ws * d)) && h->alloc(&h->ssgu, std::max<size_t>(1, L * 2 * ws)) &&
             h->alloc(&h->wsd8, std::max<size_t>(1, L * d * nsh * h->wpad)) && h->alloc(&h->ssd, L * d) &&
             h->alloc(&h->xperm8, RK * d) && h->alloc(&h->sxperm8, RK) && h->alloc(&h->xn8, R * d) &&
             h->alloc(&h->sxn8, R) && h->alloc(&h->act8, RK * w) && h->alloc(&h->sact8, RK) &&
             h->alloc(&h->actsh8, std::max<size_t>(1, R * nsh * h->wpad)) && h->alloc(&h->sactsh8, R);
    }
    h->sc = c.self_cond_width > 0;
    if (ok && h->sc) {
        const size_t rc = static_cast<size_t>(B) * C, V = c.vocab, ws = c.self_cond_width;
        const int m_tiles = static_cast<int>((rc + tc::BM - 1) / tc::BM);
        h->sc_norm = static_cast<const uint16_t*>(weights->sc_norm);
        h->sc_bn_pe = d % 256 == 0 ? 256 : 128;
        h->sc_pairs = d % 256 == 0;
        h->sc_ks = h->sc_pairs
                       ? sc_pe_splits(static_cast<int>((rc + 255) / 256) * (d / 256), c.vocab / tc::BK,
                                      h->num_sms / 2, static_cast<double>(rc) * d * sizeof(float),
                                      2.0 * (tc::BM + 128) * tc::BK * 2)
                       : sc_pe_splits(m_tiles * (d / h->sc_bn_pe), c.vocab / tc::BK, h->num_sms,
                                      static_cast<double>(rc) * d * sizeof(float),
                                      static_cast<double>(tc::BM + h->sc_bn_pe) * tc::BK * 2);
        h->sc_bn_gu = m_tiles * static_cast<int>(2 * ws / 128) >= h->num_sms ? 128 : 64;
        h->sc_kz = std::min(kMaxParts, k_splits_for(m_tiles * (d / 128), static_cast<int>(ws / tc::BK), h->num_sms));
        {
            const int num_kb = static_cast<int>(ws / tc::BK), per = (num_kb + h->sc_kz - 1) / h->sc_kz;
            h->sc_kz = (num_kb + per - 1) / per;  // every split non-empty
        }
        int sl = 1;  // p0_hat blocks per row: about 4 blocks per SM in all
        while (sl < 64 && static_cast<size_t>(sl) * rc < 4u * static_cast<size_t>(h->num_sms)) sl *= 2;
        h->sc_slices = sl;
        ok = h->alloc(&h->sc_logits, rc * V) && h->alloc(&h->sc_p, rc * V) &&
             h->alloc(&h->sc_u, static_cast<size_t>(h->sc_ks) * rc * d) && h->alloc(&h->sc_n, rc * d) &&
             h->alloc(&h->sc_act, rc * ws) && h->alloc(&h->sc_z, static_cast<size_t>(h->sc_kz) * rc * d);
    }
    if (!ok) {
        free_all(h);
        delete h;
        return DGEN_ENOMEM;
    }
    // RoPE table (cos, sin) of angle pos * base^(-2j/hd), computed in double.
    {
        std::vector<float2> tab(static_cast<size_t>(h->S_max) * (hd / 2));
        for (int p = 0; p < h->S_max; ++p)
            for (int j = 0; j < hd / 2; ++j) {
                const double ang = p * std::pow(static_cast<double>(c.rope_base), -2.0 * j / hd);
                tab[static_cast<size_t>(p) * (hd / 2) + j] = make_float2(static_cast<float>(std::cos(ang)),
                                                                         static_cast<float>(std::sin(ang)));
            }
        if (cudaMemcpy(h->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess ||
            cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess ||
            // key rows past S are read (and masked) by the 64-key attention tiles: keep them finite
            cudaMemset(h->kc, 0, h->kv_layer * c.n_layers * sizeof(bf16)) != cudaSuccess ||
            cudaMemset(h->vc, 0, h->kv_layer * c.n_layers * sizeof(bf16)) != cudaSuccess ||
            cudaMemset(h->committed, 0, static_cast<size_t>(B) * C) != cudaSuccess ||
            cudaMemset(h->eb_done, 0, B) != cudaSuccess ||
            // routing outputs read by the expert GEMMs and the combine: start in bounds
            cudaMemset(h->inv, 0, RK * sizeof(int)) != cudaSuccess ||
            cudaMemset(h->n_chunks, 0, sizeof(int)) != cudaSuccess ||
            cudaHostAlloc(reinterpret_cast<void**>(&h->host_flags), std::max(B, 1), cudaHostAllocDefault) !=
                cudaSuccess ||
            cudaMemset(h->tok, 0, static_cast<size_t>(B) * C * sizeof(int32_t)) != cudaSuccess ||
            (h->sc && cudaMemset(h->sc_z, 0, h->sc_z_bytes()) != cudaSuccess)) {
            free_all(h);
            delete h;
            return DGEN_ECUDA;
        }
    }
    // tensor maps
    const int qkv_rows = (c.n_q_heads + 2 * c.n_kv_heads) * hd;
    ok = make_map(&h->map_xn_a, h->xn, R, d, 128) && make_map(&h->map_attn_a, h->attn, R, c.n_q_heads * hd, 128) &&
         make_map(&h->map_q_attn, h->q, static_cast<uint64_t>(B) * c.n_q_heads * std::max(C, c.prompt_max), hd, 128) &&
         make_map(&h->map_embed_b, h->embed, c.vocab, d, 256) &&
         make_map(&h->map_embed_b128, h->embed, c.vocab, d, 128);
    for (int i = 0; i < 5 && ok; ++i) {
        const uint32_t br = 16u << i;
        ok = make_map(&h->map_xperm_c[i], h->xperm, RK, d, br) &&
             make_map(&h->map_act_c[i], h->act, RK, c.expert_width, br) &&
             make_map(&h->map_xn_c[i], h->xn, R, d, br) &&
             make_map(&h->map_actsh_c[i], h->act_sh, R, std::max(c.shared_width, 64), br);
    }
    if (ok && h->sc) {
        const uint64_t rc = static_cast<uint64_t>(B) * C, ws = c.self_cond_width;
        ok = make_map(&h->map_sc_p, h->sc_p, rc, c.vocab, 128) &&
             make_map(&h->map_embed_mn, h->embed, c.vocab, d, 64) &&  // 64 x 64 boxes: the MN-major B of p0_hat E
             make_map(&h->map_sc_n, h->sc_n, rc, d, 128) &&
             make_map(&h->map_sc_wgu, weights->w_sc_gate_up, 2 * ws, d, h->sc_bn_gu) &&
             make_map(&h->map_sc_act, h->sc_act, rc, ws, 128) &&
             make_map(&h->map_sc_wd, weights->w_sc_down, d, ws, 128);
    }
    h->maps.resize(c.n_layers);
    for (int l = 0; l < c.n_layers && ok; ++l) {
        const dgen_layer_weights& w = h->layers[l];
        LayerMaps& m = h->maps[l];
        ok = make_map(&m.kc, h->kc_l(l), static_cast<uint64_t>(B) * c.n_kv_heads * h->S_max, hd, 64) &&
             make_map(&m.vc, h->vc_l(l), static_cast<uint64_t>(B) * c.n_kv_heads * h->S_max, hd, 64) &&
             make_map(&m.wqkv, w.w_qkv, qkv_rows, d, hd) &&
             make_map(&m.wqkv_pair, w.w_qkv, qkv_rows, d, 64) &&
             make_map(&m.wo, w.w_o, d, c.n_q_heads * hd, 128) &&
             make_map(&m.wr, w.w_router, c.n_experts, d, h->bn_router) &&
             make_map(&m.wgu, w.w_gate_up, static_cast<uint64_t>(c.n_experts) * 2 * c.expert_width, d, 128) &&
             make_map(&m.wd, w.w_down, static_cast<uint64_t>(c.n_experts) * d, c.expert_width, 128);
        if (ok && c.shared_width > 0)
            ok = make_map(&m.wsgu, w.w_shared_gate_up, 2 * c.shared_width, d, 128) &&
                 make_map(&m.wsd, w.w_shared_down, d, c.shared_width, 128);
    }
    if (ok && h->fp8) {  // E4M3 copies of the expert weights (synchronous, once) and their maps
        const size_t E = c.n_experts, w = c.expert_width, ws = c.shared_width;
        const int nsh = h->n_shared_parts;
        auto quant = [&](const void* src, size_t rows, int cols, uint8_t* dst, size_t dst_ld, int slice, int pad,
                         float* sc) {
            quant_rows_e4m3_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256>>>(
                static_cast<const bf16*>(src), static_cast<size_t>(cols), static_cast<int>(rows), cols, dst, dst_ld,
                slice, pad, sc);
            return cudaGetLastError() == cudaSuccess;
        };
        ok = cudaMemset(h->wsd8, 0, std::max<size_t>(1, c.n_layers * static_cast<size_t>(d) * nsh * h->wpad)) ==
                 cudaSuccess &&
             cudaMemset(h->actsh8, 0, std::max<size_t>(1, R * nsh * h->wpad)) == cudaSuccess;
        for (int l = 0; l < c.n_layers && ok; ++l) {
            const dgen_layer_weights& lw = h->layers[l];
            LayerMaps& m = h->maps[l];
            uint8_t* gu8 = h->wgu8 + l * E * 2 * w * d;
            uint8_t* d8 = h->wd8 + l * E * d * w;
            ok = quant(lw.w_gate_up, E * 2 * w, d, gu8, d, d, d, h->sgu + l * E * 2 * w) &&
                 quant(lw.w_down, E * d, static_cast<int>(w), d8, w, static_cast<int>(w), static_cast<int>(w),
                       h->sd + l * E * d) &&
                 make_map_u8(&m.wgu8, gu8, E * 2 * w, d, 128) && make_map_u8(&m.wd8, d8, E * d, w, 128);
            if (ok && ws > 0) {
                uint8_t* sgu8 = h->wsgu8 + l * 2 * ws * d;
                uint8_t* sd8 = h->wsd8 + l * static_cast<size_t>(d) * nsh * h->wpad;
                ok = quant(lw.w_shared_gate_up, 2 * ws, d, sgu8, d, d, d, h->ssgu + l * 2 * ws) &&
                     quant(lw.w_shared_down, d, static_cast<int>(ws), sd8, static_cast<size_t>(nsh) * h->wpad,
                           static_cast<int>(w), h->wpad, h->ssd + l * static_cast<size_t>(d)) &&
                     make_map_u8(&m.wsgu8, sgu8, 2 * ws, d, 128) &&
                     make_map_u8(&m.wsd8, sd8, d, static_cast<uint64_t>(nsh) * h->wpad, 128);
            }
        }
        for (int i = 0; i < 5 && ok; ++i) {
            const uint32_t br = 16u << i;
            ok = make_map_u8(&h->map_xperm8_c[i], h->xperm8, RK, d, br) &&
                 make_map_u8(&h->map_act8_c[i], h->act8, RK, w, br) &&
                 make_map_u8(&h->map_xn8_c[i], h->xn8, R, d, br) &&
                 (ws == 0 || make_map_u8(&h->map_actsh8_c[i], h->actsh8, R, static_cast<uint64_t>(nsh) * h->wpad, br));
        }
        ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    }
    if (!ok) {
        free_all(h);
        delete h;
        return DGEN_EINVAL;
    }
    *out = h;
    return DGEN_OK;
}

int dgen_destroy(dgen_handle* h) {
    if (!h) return DGEN_OK;
    cudaStreamSynchronize(h->stream);
    release_graph(h);
    for (const auto& p : h->timed) {
        cudaEventDestroy(p.a);
        cudaEventDestroy(p.b);
    }
    for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
    free_all(h);
    delete h;
    return DGEN_OK;
}

int dgen_prefill_prompt(dgen_handle* h, const int32_t* prompt_dev, int32_t P) {
    if (!h || !prompt_dev || P < 1) return DGEN_EINVAL;
    if (P > h->cfg.prompt_max) return DGEN_ECAP;
    const int rows = h->cfg.batch * P;
    h->P = -1;
    DGEN_TRY(embed(h, prompt_dev, rows));
    for (int l = 0; l < h->cfg.n_layers; ++l) DGEN_TRY(run_layer(h, l, rows, P, 0, P, true, next_norm_of(h, l)));
    h->P = P;
    h->blocks_done = 0;
    std::fill(h->kv_P.begin(), h->kv_P.end(), P);
    return sc_clear(h);
}

int dgen_append_canvas(dgen_handle* h) {
    if (!h) return DGEN_EINVAL;
    if (h->P < 1) return DGEN_ESTATE;
    const dgen_config& c = h->cfg;
    const int P = h->P;
    if (P + c.canvas > c.prompt_max) return DGEN_ECAP;
    const int rows = h->rows_c;
    h->P = -1;
    DGEN_TRY(embed(h, h->tok, rows));
    for (int l = 0; l < c.n_layers; ++l)
        DGEN_TRY(run_layer(h, l, rows, c.canvas, P, P + c.canvas, true, next_norm_of(h, l)));
    h->P = P + c.canvas;
    h->blocks_done += 1;
    std::fill(h->kv_P.begin(), h->kv_P.end(), h->P);
    return sc_clear(h);
}

int dgen_set_prompt_kv(dgen_handle* h, int32_t layer, const void* k_dev, const void* v_dev, int32_t P) {
    if (!h || !k_dev || !v_dev || P < 1 || layer < 0 || layer >= h->cfg.n_layers) return DGEN_EINVAL;
    if (P > h->cfg.prompt_max) return DGEN_ECAP;
    const dgen_config& c = h->cfg;
    const size_t row_bytes = static_cast<size_t>(P) * c.head_dim * 2;
    const size_t pitch = static_cast<size_t>(h->S_max) * c.head_dim * 2;
    const int n = c.batch * c.n_kv_heads;
    if (cudaMemcpy2DAsync(h->kc_l(layer), pitch, k_dev, row_bytes, row_bytes, n, cudaMemcpyDeviceToDevice,
                          h->stream) != cudaSuccess ||
        cudaMemcpy2DAsync(h->vc_l(layer), pitch, v_dev, row_bytes, row_bytes, n, cudaMemcpyDeviceToDevice,
                          h->stream) != cudaSuccess)
        return DGEN_ECUDA;
    h->kv_P[layer] = P;
    h->P = std::all_of(h->kv_P.begin(), h->kv_P.end(), [P](int x) { return x == P; }) ? P : -1;
    h->blocks_done = 0;
    return sc_clear(h);
}

int dgen_init_canvas(dgen_handle* h, uint64_t seed) {
    if (!h) return DGEN_EINVAL;
    const int n = h->rows_c;
    launch_h(h, init_canvas_kernel, (n + 255) / 256, 256, 0, h->tok, h->committed, h->cfg.batch, h->cfg.canvas,
             static_cast<uint32_t>(h->cfg.vocab), pos_offset(h), static_cast<uint32_t>(seed),
             static_cast<uint32_t>(seed >> 32));
    DGEN_TRY(check_launch(h));
    return sc_clear(h);
}

int dgen_set_canvas(dgen_handle* h, const int32_t* tok_dev, const uint8_t* committed_dev) {
    if (!h || !tok_dev) return DGEN_EINVAL;
    const size_t n = h->rows_c;
    if (cudaMemcpyAsync(h->tok, tok_dev, n * sizeof(int32_t), cudaMemcpyDeviceToDevice, h->stream) != cudaSuccess)
        return DGEN_ECUDA;
    const cudaError_t e = committed_dev
                              ? cudaMemcpyAsync(h->committed, committed_dev, n, cudaMemcpyDeviceToDevice, h->stream)
                              : cudaMemsetAsync(h->committed, 0, n, h->stream);
    if (e != cudaSuccess) return DGEN_ECUDA;
    return sc_clear(h);
}

int dgen_set_self_cond(dgen_handle* h, const float* z_dev_or_null) {
    if (!h) return DGEN_EINVAL;
    if (!h->sc) return z_dev_or_null ? DGEN_EINVAL : DGEN_OK;
    DGEN_TRY(sc_clear(h));
    if (!z_dev_or_null) return DGEN_OK;
    const size_t bytes = static_cast<size_t>(h->rows_c) * h->cfg.d_model * sizeof(float);
    return cudaMemcpyAsync(h->sc_z, z_dev_or_null, bytes, cudaMemcpyDeviceToDevice, h->stream) == cudaSuccess
               ? DGEN_OK
               : DGEN_ECUDA;
}

int dgen_get_canvas(const dgen_handle* h, int32_t* tok_dev, uint8_t* committed_dev) {
    if (!h) return DGEN_EINVAL;
    const size_t n = h->rows_c;
    if (tok_dev && cudaMemcpyAsync(tok_dev, h->tok, n * sizeof(int32_t), cudaMemcpyDeviceToDevice, h->stream) !=
                       cudaSuccess)
        return DGEN_ECUDA;
    if (committed_dev &&
        cudaMemcpyAsync(committed_dev, h->committed, n, cudaMemcpyDeviceToDevice, h->stream) != cudaSuccess)
        return DGEN_ECUDA;
    return DGEN_OK;
}

int dgen_denoise_step(dgen_handle* h, int32_t s, int32_t T, float* logits_dev_or_null) {
    if (!h || T < 1 || s < 0 || s >= T) return DGEN_EINVAL;
    if (logits_dev_or_null && !aligned16(logits_dev_or_null)) return DGEN_EINVAL;  // written as float4
    if (h->P < 1) return DGEN_ESTATE;
    DGEN_TRY(set_tau(h, s, T));
    const bool graphable = h->use_graph && !logits_dev_or_null && !h->cap_ids && !h->cap_logits && !h->cap_h;
    if (!graphable) return step_body(h, logits_dev_or_null);
    if (h->graph && (h->graph_P != h->P || h->graph_mask != h->timing_mask || h->graph_force != h->force_canvas))
        release_graph(h);
    if (!h->graph) {
        if (h->warm_P != h->P) {  // one eager pass first (kernel attributes, first-touch of buffers)
            h->warm_P = h->P;
            return step_body(h, nullptr);
        }
        DGEN_TRY(capture_step(h));
        if (!h->graph) return step_body(h, nullptr);  // capture unsupported on this stream
    }
    if (cudaGraphLaunch(h->graph, h->stream) != cudaSuccess) return DGEN_ECUDA;
    h->launches += h->graph_launches;
    return DGEN_OK;
}

int dgen_set_logits(dgen_handle* h, const float* logits_dev, int32_t s, int32_t T) {
    if (!h || !logits_dev || T < 1 || s < 0 || s >= T) return DGEN_EINVAL;
    DGEN_TRY(set_tau(h, s, T));
    const int warps = h->rows_c * (h->cfg.vocab / 256);
    launch_h(h, stats_from_logits_kernel, (warps + 7) / 8, 256, 0, logits_dev, h->rows_c, h->cfg.vocab,
             static_cast<const float*>(h->inv_tau), h->pmax, h->psum, h->parg, h->pent);
    return check_launch(h);
}

int dgen_sample_commit(dgen_handle* h, int32_t s, int32_t T, uint64_t seed, float* conf_dev_or_null) {
    if (!h || T < 1 || s < 0 || s >= T) return DGEN_EINVAL;
    const dgen_config& c = h->cfg;
    const int rows = h->rows_c;
    Timed t(h, DGEN_K_SAMPLER);
    launch_h(h, stats_combine_kernel, (rows + 7) / 8, 256, 0, h->pmax, h->psum, h->parg, rows, c.vocab / 256,
                                                                h->inv_tau, h->conf, h->argmax);
    DGEN_TRY(check_launch(h));
    const int m = c.commit_per_step > 0 ? c.commit_per_step : (c.canvas + T - 1) / T;
    const int threads = (c.canvas + 31) / 32 * 32;
    launch_h(h, sample_commit_kernel, c.batch, threads, 0, h->tok, h->committed, h->conf, h->argmax, c.canvas,
             static_cast<uint32_t>(c.vocab), s, s == T - 1 ? 1 : 0, m, pos_offset(h), static_cast<uint32_t>(seed),
             static_cast<uint32_t>(seed >> 32), conf_dev_or_null);
    return check_launch(h);
}

int dgen_sample_commit_eb(dgen_handle* h, const float* logits_dev_or_null, int32_t s, int32_t T_max, uint64_t seed,
                          float gamma, float stop_threshold, int32_t freeze, float* entropy_dev_or_null,
                          uint8_t* stop_dev_or_null) {
    if (!h || T_max < 1 || s < 0 || s >= T_max || !(gamma >= 0.f) || !(stop_threshold >= 0.f) ||
        (freeze != 0 && freeze != 1))
        return DGEN_EINVAL;
    if (logits_dev_or_null && !aligned16(logits_dev_or_null)) return DGEN_EINVAL;  // read as float4
    const dgen_config& c = h->cfg;
    const int rows = h->rows_c;
    Timed t(h, DGEN_K_SAMPLER);
    float* ent = entropy_dev_or_null ? entropy_dev_or_null : h->conf;
    if (logits_dev_or_null) {  // given logits: own 1/tau slot, the step's statistics untouched
        DGEN_TRY(set_tau(h, s, T_max, 1));
        launch_h(h, entropy_row_kernel, rows, 256, 0, logits_dev_or_null, rows, c.vocab,
                 static_cast<const float*>(h->inv_tau + 1), ent, h->argmax);
    } else {  // the LM head's statistics of the last dgen_denoise_step (same s, T_max)
        launch_h(h, eb_stats_combine_kernel, (rows + 7) / 8, 256, 0, static_cast<const float*>(h->pmax),
                 static_cast<const float*>(h->psum), static_cast<const float*>(h->pent),
                 static_cast<const int*>(h->parg), rows, c.vocab / 256, static_cast<const float*>(h->inv_tau), ent,
                 h->argmax);
    }
    DGEN_TRY(check_launch(h));
    const int threads = (c.canvas + 31) / 32 * 32;
    launch_h(h, eb_commit_kernel, c.batch, threads, 0, h->tok, h->committed, static_cast<const float*>(ent),
             static_cast<const int*>(h->argmax), h->eb_prev_argmax, h->eb_done, c.canvas,
             static_cast<uint32_t>(c.vocab), s, s == T_max - 1 ? 1 : 0, freeze, gamma, stop_threshold, pos_offset(h),
             static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32), stop_dev_or_null);
    return check_launch(h);
}

int dgen_generate_block_eb(dgen_handle* h, const int32_t* prompt_dev, int32_t P, int32_t T_max, uint64_t seed,
                           float gamma, float stop_threshold, int32_t freeze, int32_t* out_dev,
                           int32_t* steps_host) {
    if (!h || !out_dev || !steps_host || T_max < 1 || (prompt_dev && P < 1) || !(gamma >= 0.f) ||
        !(stop_threshold >= 0.f) || (freeze != 0 && freeze != 1))
        return DGEN_EINVAL;
    const int B = h->cfg.batch;
    if (prompt_dev)
        DGEN_TRY(dgen_prefill_prompt(h, prompt_dev, P));
    else if (h->P < 1)
        return DGEN_ESTATE;
    DGEN_TRY(dgen_init_canvas(h, seed));
    for (int b = 0; b < B; ++b) steps_host[b] = 0;
    for (int s = 0; s < T_max; ++s) {
        DGEN_TRY(dgen_denoise_step(h, s, T_max, nullptr));
        DGEN_TRY(dgen_sample_commit_eb(h, nullptr, s, T_max, seed, gamma, stop_threshold, freeze, nullptr, nullptr));
        // the host reads the per-canvas done flags before launching the next step
        if (cudaMemcpyAsync(h->host_flags, h->eb_done, B, cudaMemcpyDeviceToHost, h->stream) != cudaSuccess ||
            cudaStreamSynchronize(h->stream) != cudaSuccess)
            return DGEN_ECUDA;
        bool all = true;
        for (int b = 0; b < B; ++b) {
            if (h->host_flags[b] && steps_host[b] == 0) steps_host[b] = s + 1;
            all = all && h->host_flags[b];
        }
        if (all) break;
    }
    return dgen_get_canvas(h, out_dev, nullptr);
}

int dgen_generate(dgen_handle* h, const int32_t* prompt_dev, int32_t P, int32_t n_blocks, int32_t T, uint64_t seed,
                  int32_t* out_dev) {
    if (!h || !prompt_dev || !out_dev || T < 1 || P < 1 || n_blocks < 1) return DGEN_EINVAL;
    const dgen_config& c = h->cfg;
    if (P + static_cast<int64_t>(n_blocks - 1) * c.canvas > c.prompt_max) return DGEN_ECAP;
    DGEN_TRY(dgen_prefill_prompt(h, prompt_dev, P));
    const size_t row = static_cast<size_t>(c.canvas) * sizeof(int32_t);
    for (int j = 0; j < n_blocks; ++j) {
        DGEN_TRY(dgen_init_canvas(h, seed));
        for (int s = 0; s < T; ++s) {
            DGEN_TRY(dgen_denoise_step(h, s, T, nullptr));
            DGEN_TRY(dgen_sample_commit(h, s, T, seed, nullptr));
        }
        if (cudaMemcpy2DAsync(out_dev + static_cast<size_t>(j) * c.canvas, row * n_blocks, h->tok, row, row, c.batch,
                              cudaMemcpyDeviceToDevice, h->stream) != cudaSuccess)
            return DGEN_ECUDA;
        if (j + 1 < n_blocks) DGEN_TRY(dgen_append_canvas(h));
    }
    return DGEN_OK;
}

int dgen_generate_block(dgen_handle* h, const int32_t* prompt_dev, int32_t P, int32_t T, uint64_t seed,
                        int32_t* out_dev) {
    if (!h || !out_dev || T < 1) return DGEN_EINVAL;
    DGEN_TRY(dgen_prefill_prompt(h, prompt_dev, P));
    DGEN_TRY(dgen_init_canvas(h, seed));
    for (int s = 0; s < T; ++s) {
        DGEN_TRY(dgen_denoise_step(h, s, T, nullptr));
        DGEN_TRY(dgen_sample_commit(h, s, T, seed, nullptr));
    }
    return dgen_get_canvas(h, out_dev, nullptr);
}

int dgen_generate_block_host(dgen_handle* h, const int32_t* prompt_host, int32_t P, int32_t T, uint64_t seed,
                             int32_t* out_host) {
    if (!h || !prompt_host || !out_host || T < 1 || P < 1) return DGEN_EINVAL;
    if (P > h->cfg.prompt_max) return DGEN_ECAP;
    const size_t np = static_cast<size_t>(h->cfg.batch) * P;
    if (cudaMemcpyAsync(h->prompt_buf, prompt_host, np * sizeof(int32_t), cudaMemcpyHostToDevice, h->stream) !=
        cudaSuccess)
        return DGEN_ECUDA;
    DGEN_TRY(dgen_prefill_prompt(h, h->prompt_buf, P));
    DGEN_TRY(dgen_init_canvas(h, seed));
    for (int s = 0; s < T; ++s) {
        DGEN_TRY(dgen_denoise_step(h, s, T, nullptr));
        DGEN_TRY(dgen_sample_commit(h, s, T, seed, nullptr));
    }
    if (cudaMemcpyAsync(out_host, h->tok, static_cast<size_t>(h->rows_c) * sizeof(int32_t), cudaMemcpyDeviceToHost,
                        h->stream) != cudaSuccess)
        return DGEN_ECUDA;
    return dgen_synchronize(h);
}

int dgen_forward_noise(dgen_handle* h, const int32_t* x0_dev, float kappa, uint64_t seed, int32_t step,
                       int32_t* xt_dev) {
    if (!h || !x0_dev || !xt_dev || !(kappa >= 0.f && kappa <= 1.f) || step < 0) return DGEN_EINVAL;
    const uint64_t thr = static_cast<uint64_t>(std::floor(static_cast<double>(kappa) * 4294967296.0));
    const int n = h->rows_c;
    launch_h(h, forward_noise_kernel, (n + 255) / 256, 256, 0, 
        x0_dev, xt_dev, h->cfg.batch, h->cfg.canvas, static_cast<uint32_t>(h->cfg.vocab), step, thr,
        static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
    return check_launch(h);
}

int dgen_synchronize(dgen_handle* h) {
    if (!h) return DGEN_EINVAL;
    if (cudaStreamSynchronize(h->stream) != cudaSuccess) return DGEN_ECUDA;
    int e = 0;
    if (cudaMemcpy(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DGEN_ECUDA;
    if (e != 0) {
        cudaMemset(h->err, 0, sizeof(int));
        return DGEN_EDEVICE;
    }
    return DGEN_OK;
}

int64_t dgen_launch_count(const dgen_handle* h) { return h ? h->launches : -1; }

int dgen_debug_read(dgen_handle* h, int32_t which, int32_t layer, void* dst_dev, uint64_t bytes) {
    if (!h || !dst_dev || layer < 0) return DGEN_EINVAL;
    if (which == 23 || which == 26) {  // one K-split partial of u or z
        const int n = which == 23 ? h->sc_ks : h->sc_kz;
        if (!h->sc || layer >= n) return DGEN_EINVAL;
        const size_t part = static_cast<size_t>(h->rows_c) * h->cfg.d_model;
        const float* src = (which == 23 ? h->sc_u : h->sc_z) + layer * part;
        return cudaMemcpyAsync(dst_dev, src, std::min<size_t>(part * sizeof(float), bytes), cudaMemcpyDeviceToDevice,
                               h->stream) == cudaSuccess
                   ? DGEN_OK
                   : DGEN_ECUDA;
    }
    if (layer >= h->cfg.n_layers) return DGEN_EINVAL;
    const dgen_config& c = h->cfg;
    const size_t R = h->rows_max;
    const void* src = nullptr;
    size_t size = 0;
    switch (which) {
        case 0: src = h->h; size = R * c.d_model * sizeof(float); break;
        case 1: src = h->xn; size = R * c.d_model * 2; break;
        case 2: src = h->q; size = static_cast<size_t>(c.batch) * c.n_q_heads * std::max(c.canvas, c.prompt_max) * c.head_dim * 2; break;
        case 3: src = h->attn; size = R * c.n_q_heads * c.head_dim * 2; break;
        case 4: src = h->kc_l(layer); size = h->kv_layer * 2; break;
        case 5: src = h->vc_l(layer); size = h->kv_layer * 2; break;
        case 6: src = h->argmax; size = static_cast<size_t>(h->rows_c) * sizeof(int); break;
        case 7: src = h->conf; size = static_cast<size_t>(h->rows_c) * sizeof(float); break;
        case 8: src = h->act; size = R * c.top_k * c.expert_width * 2; break;
        case 9: src = h->act8; size = h->fp8 ? R * c.top_k * c.expert_width : 0; break;
        case 10: src = h->sact8; size = h->fp8 ? R * c.top_k * sizeof(float) : 0; break;
        case 11: src = h->xperm8; size = h->fp8 ? R * c.top_k * c.d_model : 0; break;
        case 12: src = h->sxperm8; size = h->fp8 ? R * c.top_k * sizeof(float) : 0; break;
        case 13: src = h->perm_tok; size = R * c.top_k * sizeof(int); break;
        case 14: src = h->yperm; size = R * c.top_k * c.d_model * sizeof(float); break;
        case 15: src = h->perm_gate; size = R * c.top_k * sizeof(float); break;
        case 16: src = c.shared_width ? h->act_sh : nullptr; size = R * c.shared_width * 2; break;
        case 17: src = (h->fp8 && c.shared_width) ? h->actsh8 : nullptr; size = R * h->n_shared_parts * h->wpad; break;
        case 18: src = (h->fp8 && c.shared_width) ? h->sactsh8 : nullptr; size = R * sizeof(float); break;
        case 19: src = h->fp8 ? h->xn8 : nullptr; size = R * c.d_model; break;
        case 20: src = h->fp8 ? h->sxn8 : nullptr; size = R * sizeof(float); break;
        case 21: src = c.shared_width ? h->y_sh : nullptr; size = h->n_shared_parts * R * c.d_model * sizeof(float); break;
        case 22: src = h->sc_p; size = static_cast<size_t>(h->rows_c) * c.vocab * 2; break;
        case 24: src = h->sc_n; size = static_cast<size_t>(h->rows_c) * c.d_model * 2; break;
        case 25: src = h->sc_act; size = static_cast<size_t>(h->rows_c) * c.self_cond_width * 2; break;
        default: return DGEN_EINVAL;
    }
    if (!src || size == 0) return DGEN_EINVAL;
    return cudaMemcpyAsync(dst_dev, src, std::min<size_t>(size, bytes), cudaMemcpyDeviceToDevice, h->stream) ==
                   cudaSuccess
               ? DGEN_OK
               : DGEN_ECUDA;
}

int dgen_force_routing(dgen_handle* h, const int32_t* prompt_ids_dev, const int32_t* canvas_ids_dev) {
    if (!h) return DGEN_EINVAL;
    h->force_prompt = prompt_ids_dev;
    h->force_canvas = canvas_ids_dev;
    return DGEN_OK;
}

int dgen_expert_usage(dgen_handle* h, int32_t* touched_host) {
    if (!h || !touched_host) return DGEN_EINVAL;
    if (cudaStreamSynchronize(h->stream) != cudaSuccess ||
        cudaMemcpy(touched_host, h->touched, sizeof(int32_t) * h->cfg.n_layers, cudaMemcpyDeviceToHost) != cudaSuccess)
        return DGEN_ECUDA;
    return DGEN_OK;
}

int dgen_set_tuning(dgen_handle* h, int32_t key, int32_t value) {
    if (!h || value < 0) return DGEN_EINVAL;
    switch (key) {
        case DGEN_TUNE_EXPERT_CHUNK:
            if (value != 0 && value != 32 && value != 64 && value != 128 && value != 256) return DGEN_EINVAL;
            h->tune_chunk = value;
            break;
        case DGEN_TUNE_ATTN_SPLITS: h->tune_attn_splits = std::min(value, h->max_splits); break;
        case DGEN_TUNE_ROUTER_SPLITS: h->tune_router_splits = value; break;
        case DGEN_TUNE_QKV_SPLITS: h->tune_qkv_splits = std::min(value, 4); break;
        case DGEN_TUNE_ATTN_KERNEL:
            if (value > 1) return DGEN_EINVAL;
            h->tune_attn_kernel = value;
            break;
        case DGEN_TUNE_SEPARATE_EXPERTS:
            if (value > 1) return DGEN_EINVAL;
            h->tune_separate_experts = value;
            break;
        case DGEN_TUNE_STATIC_ITEMS:
            if (value > 1) return DGEN_EINVAL;
            h->tune_static_items = value;
            break;
        case DGEN_TUNE_PAIRS:
            if (value > 2) return DGEN_EINVAL;
            h->tune_pairs = value;
            break;
        case DGEN_TUNE_CHUNK_ORDER:
            if (value > 2) return DGEN_EINVAL;
            h->tune_chunk_order = value;
            break;
        case DGEN_TUNE_ROUTE_BARRIER_EXTRA:
            if (value > 1) return DGEN_EINVAL;
            h->route_barrier_extra = static_cast<unsigned int>(value);
            break;
        default: return DGEN_EINVAL;
    }
    release_graph(h);
    return DGEN_OK;
}

int dgen_set_flags(dgen_handle* h, uint32_t flags) {
    if (!h) return DGEN_EINVAL;
    h->use_graph = !(flags & DGEN_FLAG_NO_GRAPH);
    if (!h->use_graph) release_graph(h);
    g_pdl.store(!(flags & DGEN_FLAG_NO_PDL));
    return DGEN_OK;
}

int dgen_capture_routing(dgen_handle* h, int32_t* ids_dev, float* logits_dev) {
    if (!h) return DGEN_EINVAL;
    h->cap_ids = ids_dev;
    h->cap_logits = logits_dev;
    return DGEN_OK;
}

int dgen_capture_residual(dgen_handle* h, float* h_dev) {
    if (!h) return DGEN_EINVAL;
    h->cap_h = h_dev;
    return DGEN_OK;
}

int dgen_set_timing(dgen_handle* h, uint32_t class_mask) {
    if (!h) return DGEN_EINVAL;
    h->timing_mask = class_mask & ((1u << DGEN_K_CLASSES) - 1u);
    return DGEN_OK;
}

int dgen_get_timing(dgen_handle* h, int32_t cls, double* total_ms, int64_t* launches) {
    if (!h || cls < 0 || cls >= DGEN_K_CLASSES) return DGEN_EINVAL;
    if (cudaStreamSynchronize(h->stream) != cudaSuccess) return DGEN_ECUDA;
    for (const auto& p : h->timed) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
            h->t_ms[p.cls] += ms;
            h->t_n[p.cls] += 1;
        }
        h->ev_pool.push_back(p.a);
        h->ev_pool.push_back(p.b);
    }
    h->timed.clear();
    double ms_graph = 0.0;
    int64_t n_graph = 0;
    for (const auto& p : h->graph_pairs) {  // the captured pass: durations of its last replay
        float ms = 0.f;
        if (p.cls == cls && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
            ms_graph += ms;
            ++n_graph;
        }
    }
    cudaGetLastError();
    if (total_ms) *total_ms = h->t_ms[cls] + ms_graph;
    if (launches) *launches = h->t_n[cls] + n_graph;
    h->t_ms[cls] = 0.0;
    h->t_n[cls] = 0;
    return DGEN_OK;
}

int dgen_gemm_e4m3(const void* a_dev, const void* b_dev, float* d_dev, int32_t M, int32_t N, int32_t K,
                   void* stream) {
    if (M < 1 || N < 1 || K < 16 || K % 16 || !d_dev) return DGEN_EINVAL;
    if (!load_encode()) return DGEN_ECUDA;
    CUtensorMap ta, tb;
    if (!make_map_u8(&ta, a_dev, M, K, 128) || !make_map_u8(&tb, b_dev, N, K, 128)) return DGEN_EINVAL;
    static int* err = nullptr;
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!err && (cudaMalloc(&err, sizeof(int)) != cudaSuccess || cudaMemset(err, 0, sizeof(int)) != cudaSuccess))
            return DGEN_ECUDA;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    tc::DenseSched sc{(M + 127) / 128, (N + 127) / 128};
    EpiStoreF32 ep{d_dev, M, N, N};
    return launch_gemm<128, 1, tc::DenseSched, EpiStoreF32, 1>(static_cast<cudaStream_t>(stream), dev, err, ta, tb,
                                                                sc, ep, K, std::min(sms, sc.m_tiles * sc.n_tiles),
                                                                nullptr);
}

int dgen_gemm_bf16(const void* a_dev, const void* b_dev, float* d_dev, int32_t M, int32_t N, int32_t K,
                   void* stream) {
    if (M < 1 || N < 1 || K < 8 || K % 8 || !d_dev) return DGEN_EINVAL;
    if (!load_encode()) return DGEN_ECUDA;
    CUtensorMap ta, tb;
    if (!make_map(&ta, a_dev, M, K, 128) || !make_map(&tb, b_dev, N, K, 128)) return DGEN_EINVAL;
    static int* err = nullptr;
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!err && (cudaMalloc(&err, sizeof(int)) != cudaSuccess || cudaMemset(err, 0, sizeof(int)) != cudaSuccess))
            return DGEN_ECUDA;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    tc::DenseSched sc{(M + 127) / 128, (N + 127) / 128};
    EpiStoreF32 ep{d_dev, M, N, N};
    return launch_gemm<128, 1>(static_cast<cudaStream_t>(stream), dev, err, ta, tb, sc, ep, K,
                               std::min(sms, sc.m_tiles * sc.n_tiles), nullptr);
}

int dgen_gemm_bf16_pair(const void* a_dev, const void* b_dev, float* d_dev, int32_t M, int32_t N, int32_t K,
                        void* stream) {
    if (M < 1 || N < 1 || K < 8 || K % 8 || !d_dev) return DGEN_EINVAL;
    if (!load_encode()) return DGEN_ECUDA;
    CUtensorMap ta, tb;
    if (!make_map(&ta, a_dev, M, K, 128) || !make_map(&tb, b_dev, N, K, 128)) return DGEN_EINVAL;
    static int* err = nullptr;
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!err && (cudaMalloc(&err, sizeof(int)) != cudaSuccess || cudaMemset(err, 0, sizeof(int)) != cudaSuccess))
            return DGEN_ECUDA;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    tc2::DensePairSched sc;
    sc.m_tiles = (M + 255) / 256;
    sc.n_tiles = (N + 255) / 256;
    EpiStoreF32 ep{d_dev, M, N, N};
    return launch_gemm_pair<256>(static_cast<cudaStream_t>(stream), dev, err, ta, tb, sc, ep, K,
                                 std::min(sms / 2, sc.m_tiles * sc.n_tiles), nullptr);
}

#ifdef DGEN_PROBES
// Measurement probe (include/dgen_probe.h), compiled only into libdgen_probe.so.
int dgen_gemm_rowsum_variant(const void* a_dev, const void* b_dev, float* out_dev, int32_t M, int32_t N, int32_t K,
                             int32_t variant, void* stream) {
    static const int kBN[6] = {64, 64, 64, 32, 128, 256};
    if (M < 1 || N < 1 || K < 8 || K % 8 || !out_dev || variant < 0 || variant > 5) return DGEN_EINVAL;
    if (!load_encode()) return DGEN_ECUDA;
    const int bn = kBN[variant];
    const int a_box = variant == 1 ? 16 : 128;
    CUtensorMap ta, tb;
    if (!make_map(&ta, a_dev, M, K, a_box) || !make_map(&tb, b_dev, N, K, bn)) return DGEN_EINVAL;
    static int* err = nullptr;
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!err && (cudaMalloc(&err, sizeof(int)) != cudaSuccess || cudaMemset(err, 0, sizeof(int)) != cudaSuccess))
            return DGEN_ECUDA;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    tc::DenseSched sc{(M + 127) / 128, (N + bn - 1) / bn};
    EpiRowSum ep{out_dev, M, sc.n_tiles};
    const int grid = std::min(sms, sc.m_tiles * sc.n_tiles);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (variant) {
        case 0: return launch_gemm<64, 1>(st, dev, err, ta, tb, sc, ep, K, grid, nullptr);
        case 1: return launch_gemm<64, 8>(st, dev, err, ta, tb, sc, ep, K, grid, nullptr);
        case 2: {
            using L = tc::Layout<64, 4, 0>;
            auto kern = tc::gemm_kernel<64, 4, 1, 0, tc::DenseSched, EpiRowSum>;
            set_smem_attr_once(kern, L::SMEM_BYTES, dev);
            kern<<<grid, 192, L::SMEM_BYTES, st>>>(ta, tb, sc, ep, (K + 63) / 64, err);
            return cudaPeekAtLastError() == cudaSuccess ? DGEN_OK : DGEN_ECUDA;
        }
        case 3: return launch_gemm<32, 1>(st, dev, err, ta, tb, sc, ep, K, grid, nullptr);
        case 4: return launch_gemm<128, 1>(st, dev, err, ta, tb, sc, ep, K, grid, nullptr);
        default: return launch_gemm<256, 1>(st, dev, err, ta, tb, sc, ep, K, grid, nullptr);
    }
}
#endif  // DGEN_PROBES

}  // extern "C"

// ================================================================== allocation-free sampler entry point
// Scratch for dgen_sample_from_logits_noalloc: per-(row, 256-column tile)
// softmax statistics, per-row confidence and argmax, and 1/tau.  In host code
// the array's name is only a stand-in: its device address comes from
// cudaGetSymbolAddress, looked up once per device.

namespace {
constexpr size_t kNaMaxRows = 8192;
constexpr size_t kNaMaxTiles = 262144;  // rows * (vocab / 256)
constexpr size_t kNaOffSum = kNaMaxTiles * 4;
constexpr size_t kNaOffArg = kNaMaxTiles * 8;
constexpr size_t kNaOffConf = kNaMaxTiles * 12;
constexpr size_t kNaOffArgmax = kNaOffConf + kNaMaxRows * 4;
constexpr size_t kNaOffTau = kNaOffArgmax + kNaMaxRows * 4;
constexpr size_t kNaBytes = kNaOffTau + 256;
constexpr int kNaMaxDevices = 64;
std::mutex g_na_mu;
void* g_na_ptr[kNaMaxDevices] = {};
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaBytes];

extern "C" int dgen_sample_from_logits_noalloc(const float* logits_dev, int32_t* tok_dev, uint8_t* committed_dev,
                                               int32_t batch, int32_t canvas, int32_t vocab, int32_t s, int32_t T,
                                               uint64_t seed, float tau_max, float tau_min, int32_t commit_per_step,
                                               float* conf_dev_or_null, void* stream) {
    if (!logits_dev || !tok_dev || !committed_dev || batch < 1 || canvas < 1 || canvas > 1024 || vocab < 256 ||
        vocab % 256 || T < 1 || s < 0 || s >= T || !(tau_max > 0.f) || !(tau_min > 0.f) || commit_per_step < 0)
        return DGEN_EINVAL;
    const size_t rows = static_cast<size_t>(batch) * canvas;
    const size_t n_tiles = static_cast<size_t>(vocab) / 256;
    if (rows > kNaMaxRows || rows * n_tiles > kNaMaxTiles) return DGEN_ESCRATCH;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNaMaxDevices) return DGEN_ECUDA;
    unsigned char* base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_na_mu);
        if (!g_na_ptr[dev]) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DGEN_ECUDA;
            g_na_ptr[dev] = p;
        }
        base = static_cast<unsigned char*>(g_na_ptr[dev]);
    }
    float* pmax = reinterpret_cast<float*>(base);
    float* psum = reinterpret_cast<float*>(base + kNaOffSum);
    int* parg = reinterpret_cast<int*>(base + kNaOffArg);
    float* conf = reinterpret_cast<float*>(base + kNaOffConf);
    int* amax = reinterpret_cast<int*>(base + kNaOffArgmax);
    float* inv_tau = reinterpret_cast<float*>(base + kNaOffTau);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const double t = 1.0 - static_cast<double>(s) / T;
    const double tau = tau_min + (static_cast<double>(tau_max) - tau_min) * t;
    set_inv_tau_kernel<<<1, 1, 0, st>>>(inv_tau, static_cast<float>(1.4426950408889634 / tau));
    const int r = static_cast<int>(rows), nt = static_cast<int>(n_tiles);
    const int warps = r * nt;
    stats_from_logits_kernel<<<(warps + 7) / 8, 256, 0, st>>>(logits_dev, r, vocab, inv_tau, pmax, psum, parg,
                                                              nullptr);
    stats_combine_kernel<<<(r + 7) / 8, 256, 0, st>>>(pmax, psum, parg, r, nt, inv_tau, conf, amax);
    const int m = commit_per_step > 0 ? commit_per_step : (canvas + T - 1) / T;
    sample_commit_kernel<<<batch, (canvas + 31) / 32 * 32, 0, st>>>(
        tok_dev, committed_dev, conf, amax, canvas, static_cast<uint32_t>(vocab), s, s == T - 1 ? 1 : 0, m, 0u,
        static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32), conf_dev_or_null);
    return cudaPeekAtLastError() == cudaSuccess ? DGEN_OK : DGEN_ECUDA;
}
