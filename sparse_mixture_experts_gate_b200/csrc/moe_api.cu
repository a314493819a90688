// moe_api.cu - the C ABI declared in include/moe.h: argument validation, the
// workspace plan, TMA descriptors, and the launch sequence of one MoE layer
// forward (router -> dispatch -> row scatter -> expert GEMM 1 -> expert GEMM 2 ->
// combine) and of its statistics.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "moe.h"
#include "moe_common.cuh"
#include "moe_kernels.cuh"

using namespace moe;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Row-major bf16 matrix [rows][inner] read in boxes of 64 x box_rows with 128B
// swizzle (the layout the UMMA shared-memory descriptors expect).
// Row-major bf16 [rows][inner] operand map: box of 64 elements (128 bytes) x
// box_rows, 128B swizzle (the UMMA K-major layout).
bool encode_bf16_2d(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows == 0) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major bf16 [rows][inner] output map for the expert GEMM's stores: box of
// 128 x 32 elements (32 rows of 256 bytes), no swizzle.
bool encode_bf16_store(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows == 0) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {128, 32};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Plan {
    int T = 0;
    int64_t C = 0;
    int T_pad = 0, n_stat_chunks = 0, n_chunks = 0, R_routed_max = 0, R_max = 0, max_row_blocks = 0;
    int max_tok_tiles = 0, max_narrow_tiles = 0;
    int n_tile_done = 0;  // per-token-tile counters of the two-layer expert GEMM launch
    int ksplit = 1, n_mtiles = 0;  // the fused router's K splits and token tiles
    size_t o_lpart = 0, ctrl_bytes = 0;
    size_t o_ctrl, o_rcnt, o_logits, o_idx, o_gates, o_slot, o_rowof, o_lse, o_psum, o_ccount, o_cbase, o_cpre, o_ckept,
        o_gstart, o_grows, o_bgroup, o_toktiles, o_narrowtiles, o_tiledone, o_rowassign, o_wsplit, o_xp, o_h, o_o, o_credit, o_partials,
        o_prestart, o_gsorted, o_rownorm, o_gz;
    size_t total = 0;
};

}  // namespace

namespace moe {
// Records `msg` as the calling thread's last error (for moe_last_error) and
// returns `code`; used by entry points defined in other files.
int report_error(int code, const char *msg) { return fail(code, "%s", msg); }
}  // namespace moe

struct moe_layer {
    moe_config_t cfg;
    moe_weights_t w;
    int G = 0;         // groups in the weight stacks: routed experts held here + shared
    int E_weights = 0; // routed experts held in the weight stacks (E, or E / ep_size)
    bool tc = false;
    int num_sms = 148;
    int num_pairs = 0;  // co-resident 2-CTA clusters of the expert GEMM
    int router_pairs = 0;  // and of the fused router
    int selftest_skip_stage = -1;  // moe_selftest_gemm_timeout only: GEMM 1's skipped stage
    int selftest_router_skip = -1;  // moe_selftest_router_timeout only: the fused router's skipped stage
    void *planes = nullptr;        // moe_prepare_router's persistent bf16 planes of the router matrix, or null
    CUtensorMap map_w1, map_w2;
    CUtensorMap map_w1h, map_w2h;  // the same with boxes of 64 rows (transposed last feature tiles)
    // State of the most recent forward, read by moe_aux_stats.
    bool has_forward = false;
    Plan plan;
    char *ws = nullptr;
    int fwd_launches = 0, stats_launches = 0;
    const void *fx = nullptr;  // the forward's tokens and gates, for the later phases
    float *fgates = nullptr;
    bool timing = false;
    cudaEvent_t ev[MOE_TIMING_EVENTS];
};

namespace {

int64_t capacity_of(const moe_config_t &c, int T) {
    if (c.capacity_factor <= 0.f) return T;
    return (int64_t)std::ceil((double)c.capacity_factor * (double)c.num_active * (double)T / (double)c.num_experts);
}

// The expert GEMMs run narrow units (token tiles of at most kNarrowTile rows,
// a deeper pipeline of weight tiles) when the experts' segments average at
// most kNarrowTile rows: there the GEMMs stream the weights and the token
// tiles are short anyway (decode-sized batches).
bool narrow_gemm(const moe_layer *L, int T) {
    const moe_config_t &c = L->cfg;
    return L->tc && (int64_t)c.num_active * T <= (int64_t)kNarrowTile * c.num_experts;
}

Plan make_plan(const moe_layer &L, int T) {
    const moe_config_t &c = L.cfg;
    Plan p;
    p.T = T;
    p.C = capacity_of(c, T);
    const int E = c.num_experts, k = c.num_active, S = c.num_shared;
    const int64_t kept_max = std::min<int64_t>((int64_t)k * T, (int64_t)E * p.C);
    const int64_t routed = std::min<int64_t>(round_up(kept_max + (int64_t)E * (kRowBlock - 1), kRowBlock),
                                             (int64_t)E * round_up(p.C, kRowBlock));
    p.R_routed_max = (int)routed;
    p.T_pad = (int)round_up(T, kRowBlock);
    p.R_max = p.R_routed_max + S * p.T_pad;
    p.max_row_blocks = p.R_max / kRowBlock;
    // Each expert's segment splits into ceil(rows / 256) token tiles of >= 32 rows.
    p.max_tok_tiles = (int)std::min<int64_t>(routed / kTokTile + E, routed / kRowBlock) +
                      S * (int)((p.T_pad + kTokTile - 1) / kTokTile);
    p.max_narrow_tiles = (int)std::min<int64_t>(routed / kNarrowTile + E, routed / kRowBlock) +
                         S * (int)((p.T_pad + kNarrowTile - 1) / kNarrowTile);
    // bf16 linear routers route in the fused tensor-core kernel (a P-sum row
    // per CTA of its launch); the MLP gate and fp32 layers route in the
    // CUDA-core router kernel.
    const bool fused_routes = c.dtype == MOE_DTYPE_BF16 && !c.use_mlp_gater;
    const int E_tc = c.use_mlp_gater ? c.gater_hidden_dim : E;  // rows of the tensor-core router matrix
    const bool tc = c.dtype == MOE_DTYPE_BF16;
    p.n_mtiles = tc ? router_fused_mtiles(T) : 0;
    p.ksplit = tc ? router_fused_ksplit(T, E_tc, c.input_dim, L.router_pairs) : 1;
    const int pieces = tc ? p.ksplit * (router_fused_epad(E_tc) / router_fused_bn(E_tc)) : 1;
    p.n_stat_chunks = fused_routes ? router_fused_ctas(p.n_mtiles * pieces, L.router_pairs) : router_psum_blocks(T);
    const int64_t n_items = c.capacity_priority == MOE_PRIORITY_RANK ? (int64_t)k * T : T;
    p.n_chunks = (int)((n_items + 255) / 256);
    const size_t es = c.dtype == MOE_DTYPE_BF16 ? 2 : 4;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    p.o_ctrl = take(kCtrlWords * 4);
    p.o_rcnt = take(16);                           // the fused router's grid-barrier counter
    p.ctrl_bytes = off - p.o_ctrl;                // control words and counters: zeroed every forward
    p.o_logits = take((size_t)T * E * 4);
    p.o_idx = take((size_t)T * k * 4);
    p.o_gates = take((size_t)T * k * 4);
    p.o_slot = take((size_t)T * k * 4);
    p.o_rowof = take((size_t)T * k * 4);
    p.o_lse = take((size_t)T * 4);
    p.o_psum = take((size_t)p.n_stat_chunks * E * 4);
    p.o_ccount = take((size_t)p.n_chunks * E * 4);
    p.o_cbase = take((size_t)p.n_chunks * E * 4);
    p.o_cpre = take((size_t)E * 4);
    p.o_ckept = take((size_t)E * 4);
    p.o_gstart = take((size_t)(E + S + 1) * 4);
    p.o_grows = take((size_t)(E + S) * 4);
    p.o_bgroup = take((size_t)p.max_row_blocks * 4);
    p.o_toktiles = take((size_t)std::max(p.max_tok_tiles, 1) * 16);
    p.o_narrowtiles = take((size_t)std::max(p.max_narrow_tiles, 1) * 16);
    p.n_tile_done = std::max(std::max(p.max_tok_tiles, p.max_narrow_tiles), 1);
    p.o_tiledone = take((size_t)p.n_tile_done * 4);
    p.o_rowassign = take((size_t)p.R_max * 4);
    p.o_partials = take((size_t)(4 * E + 3) * 4);
    p.o_prestart = take((size_t)E * 4);
    p.o_gsorted = take((size_t)T * k * 4);
    p.o_rownorm = take(c.credit_norm == MOE_CREDIT_HIDDEN ? (size_t)p.R_routed_max * 4 : 0);
    p.o_credit = take((size_t)T * k * 4);
    p.o_wsplit = take(tc ? (size_t)router_fused_epad(E_tc) * 3 * c.input_dim * 2 : 0);
    p.o_gz = take(c.use_mlp_gater ? (size_t)T * c.gater_hidden_dim * 4 : 0);
    p.o_lpart = take(pieces > 1 ? (size_t)p.n_mtiles * 256 * router_fused_epad(E_tc) * p.ksplit * 4 : 0);
    p.o_xp = take(c.dtype == MOE_DTYPE_BF16 ? (size_t)p.R_routed_max * c.input_dim * es : 0);
    p.o_h = take((size_t)p.R_max * c.expert_dim * es);
    p.o_o = take((size_t)p.R_max * c.output_dim * es);
    p.total = off;
    return p;
}

int validate_config(const moe_config_t *c, const moe_weights_t *w) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
    if (!w) return fail(MOE_ERR_INVALID_ARG, "weights is NULL");
    if (c->num_experts < 1) return fail(MOE_ERR_INVALID_ARG, "num_experts must be >= 1 (got %d)", c->num_experts);
    if (c->num_experts > 256)
        return fail(MOE_ERR_UNSUPPORTED, "num_experts > 256 is not supported (got %d)", c->num_experts);
    if (c->num_active < 1 || c->num_active > c->num_experts)
        return fail(MOE_ERR_INVALID_ARG, "num_active must be in 1..num_experts (got %d, E=%d)", c->num_active,
                    c->num_experts);
    if (c->num_active > 16) return fail(MOE_ERR_UNSUPPORTED, "num_active > 16 is not supported");
    if (c->input_dim < 1 || c->expert_dim < 1 || c->output_dim < 1)
        return fail(MOE_ERR_INVALID_ARG, "input_dim, expert_dim and output_dim must be >= 1");
    if (c->num_shared < 0) return fail(MOE_ERR_INVALID_ARG, "num_shared must be >= 0");
    if (c->num_shared > 4) return fail(MOE_ERR_UNSUPPORTED, "num_shared > 4 is not supported");
    if (c->activation < MOE_ACT_RELU || c->activation > MOE_ACT_SWISH)
        return fail(MOE_ERR_INVALID_ARG, "unknown activation %d", c->activation);
    if (c->top_k_method != MOE_TOPK_GREEDY && c->top_k_method != MOE_TOPK_NOISY)
        return fail(MOE_ERR_INVALID_ARG, "unknown top_k_method %d", c->top_k_method);
    if (c->dtype != MOE_DTYPE_BF16 && c->dtype != MOE_DTYPE_FP32)
        return fail(MOE_ERR_INVALID_ARG, "unknown dtype %d", c->dtype);
    if (c->max_tokens < 0) return fail(MOE_ERR_INVALID_ARG, "max_tokens must be >= 0");
    if (!(c->temperature == 1.0f))
        return fail(MOE_ERR_UNSUPPORTED, "router temperature other than 1 is not supported");
    if (c->capacity_factor != c->capacity_factor) return fail(MOE_ERR_INVALID_ARG, "capacity_factor is NaN");
    if (c->credit_norm != MOE_CREDIT_OUTPUT && c->credit_norm != MOE_CREDIT_HIDDEN)
        return fail(MOE_ERR_INVALID_ARG, "unknown credit_norm %d", c->credit_norm);
    if (c->capacity_priority != MOE_PRIORITY_TOKEN && c->capacity_priority != MOE_PRIORITY_RANK)
        return fail(MOE_ERR_INVALID_ARG, "unknown capacity_priority %d", c->capacity_priority);
    if (c->ep_size < 1 || c->ep_rank < 0 || c->ep_rank >= c->ep_size)
        return fail(MOE_ERR_INVALID_ARG, "ep_size must be >= 1 and 0 <= ep_rank < ep_size (got %d, %d)", c->ep_size,
                    c->ep_rank);
    if (c->ep_size > 1) {
        if (c->num_experts % c->ep_size)
            return fail(MOE_ERR_INVALID_ARG, "num_experts (%d) must be a multiple of ep_size (%d)", c->num_experts,
                        c->ep_size);
        if (c->dtype != MOE_DTYPE_BF16)
            return fail(MOE_ERR_UNSUPPORTED, "expert parallelism runs bf16 layers (tensor-core expert GEMMs)");
        if (c->credit_norm == MOE_CREDIT_HIDDEN)
            return fail(MOE_ERR_UNSUPPORTED, "the hidden-activation credit needs the hidden rows on the token's rank");
    }
    if (c->use_mlp_gater != 0 && c->use_mlp_gater != 1)
        return fail(MOE_ERR_INVALID_ARG, "use_mlp_gater must be 0 or 1");
    if (c->use_mlp_gater) {
        if (c->gater_hidden_dim < 1 || c->gater_hidden_dim > 256)
            return fail(MOE_ERR_UNSUPPORTED, "gater_hidden_dim must be in 1..256 (got %d)", c->gater_hidden_dim);
        if (!w->gater_w1) return fail(MOE_ERR_INVALID_ARG, "use_mlp_gater is set but weights->gater_w1 is NULL");
    }
    if (!w->w_gate) return fail(MOE_ERR_INVALID_ARG, "weights->w_gate is NULL");
    if (!w->w1) return fail(MOE_ERR_INVALID_ARG, "weights->w1 is NULL");
    if (!w->w2) return fail(MOE_ERR_INVALID_ARG, "weights->w2 is NULL");
    if (c->use_selection_bias && !w->sel_bias)
        return fail(MOE_ERR_INVALID_ARG, "use_selection_bias is set but weights->sel_bias is NULL");
    if (c->dtype == MOE_DTYPE_BF16) {
        if (c->input_dim % 64 || c->expert_dim % 64 || c->output_dim % 64)
            return fail(MOE_ERR_UNSUPPORTED, "bf16 layers need input_dim, expert_dim and output_dim multiples of 64");
    } else {
        if (c->input_dim % 4 || c->expert_dim % 4 || c->output_dim % 4)
            return fail(MOE_ERR_UNSUPPORTED, "fp32 layers need input_dim, expert_dim, output_dim multiples of 4");
    }
    return MOE_OK;
}

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

#define MOE_MARK(L, i, s)                                                                       \
    do {                                                                                        \
        if ((L)->timing) MOE_LAUNCH(cudaEventRecord((L)->ev[i], s));                            \
    } while (0)

#define MOE_LAUNCH(expr)                                                                              \
    do {                                                                                              \
        cudaError_t e_ = (expr);                                                                      \
        if (e_ != cudaSuccess) return fail(MOE_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_)); \
    } while (0)

}  // namespace

extern "C" {

moe_config_t moe_config_default(void) {
    moe_config_t c;
    std::memset(&c, 0, sizeof c);
    c.num_experts = 8;
    c.num_active = 2;
    c.input_dim = 512;
    c.expert_dim = 1024;
    c.output_dim = 512;
    c.num_shared = 0;
    c.capacity_factor = 1.25f;
    c.activation = MOE_ACT_GELU;
    c.top_k_method = MOE_TOPK_GREEDY;
    c.use_selection_bias = 0;
    c.dtype = MOE_DTYPE_BF16;
    c.max_tokens = 0;
    c.load_balance_coef = 0.01f;
    c.z_loss_coef = 1e-3f;
    c.temperature = 1.0f;
    c.credit_norm = MOE_CREDIT_OUTPUT;
    c.capacity_priority = MOE_PRIORITY_TOKEN;
    c.use_mlp_gater = 0;
    c.gater_hidden_dim = 128;
    c.ep_size = 1;
    c.ep_rank = 0;
    return c;
}

int moe_layer_create(const moe_config_t *cfg, const moe_weights_t *w, moe_layer_t **out) {
    g_last_error.clear();
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    int rc = validate_config(cfg, w);
    if (rc != MOE_OK) return rc;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10 || minor != 0)
        return fail(MOE_ERR_CUDA, "device %d is sm_%d%d; this library is built for sm_100a", dev, major, minor);
    moe_layer *L = new moe_layer();
    L->cfg = *cfg;
    L->w = *w;
    L->E_weights = cfg->num_experts / (cfg->ep_size > 1 ? cfg->ep_size : 1);
    L->G = L->E_weights + cfg->num_shared;
    L->num_sms = sms > 0 ? sms : 148;
    L->tc = cfg->dtype == MOE_DTYPE_BF16;
    if (L->tc) {
        if (!encode_bf16_2d(&L->map_w1, w->w1, cfg->input_dim, (uint64_t)L->G * cfg->expert_dim, 128) ||
            !encode_bf16_2d(&L->map_w2, w->w2, cfg->expert_dim, (uint64_t)L->G * cfg->output_dim, 128) ||
            !encode_bf16_2d(&L->map_w1h, w->w1, cfg->input_dim, (uint64_t)L->G * cfg->expert_dim, 64) ||
            !encode_bf16_2d(&L->map_w2h, w->w2, cfg->expert_dim, (uint64_t)L->G * cfg->output_dim, 64)) {
            delete L;
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the expert weights (16-byte alignment?)");
        }
        L->num_pairs = gemm_pair_max_pairs(L->num_sms);
        L->router_pairs = router_fused_max_pairs(L->num_sms);
        if (L->num_pairs <= 0 || L->router_pairs <= 0) {
            delete L;
            return fail(MOE_ERR_CUDA, "no 2-CTA cluster of the expert GEMM or router fits on device %d", dev);
        }
    }
    *out = L;
    return MOE_OK;
}

size_t moe_workspace_bytes(const moe_layer_t *layer, int32_t T) {
    if (!layer || T < 0) return 0;
    return make_plan(*layer, T).total;
}

int64_t moe_capacity(const moe_layer_t *layer, int32_t T) {
    if (!layer || T < 0) return -1;
    return capacity_of(layer->cfg, T);
}

}  // extern "C"

namespace {

// Router, dispatch and row scatter of one forward (everything before the
// expert GEMMs); records what the later phases need in the layer.
int fwd_route(moe_layer_t *L, const void *x, int32_t T, const float *logit_noise, void *workspace, size_t ws_bytes,
              const moe_routing_t *routing, cudaStream_t s,
              bool router_only = false) {
    const moe_config_t &c = L->cfg;
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0 (got %d)", T);
    if (c.max_tokens > 0 && T > c.max_tokens)
        return fail(MOE_ERR_INVALID_ARG, "T=%d exceeds max_tokens=%d", T, c.max_tokens);
    if (T > 0 && !x) return fail(MOE_ERR_INVALID_ARG, "x is required when T > 0");
    if (T > 0 && c.top_k_method == MOE_TOPK_NOISY && !logit_noise)
        return fail(MOE_ERR_INVALID_ARG, "NOISY top-k needs logit_noise [T][E]");
    const Plan p = make_plan(*L, T);
    if (!workspace) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(workspace) % 256)
        return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (ws_bytes < p.total)
        return fail(MOE_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed for T=%d", ws_bytes, p.total, T);
    if (reinterpret_cast<uintptr_t>(x) % 16) return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");

    char *ws = static_cast<char *>(workspace);
    L->has_forward = true;
    L->plan = p;
    L->ws = ws;
    L->fwd_launches = 0;
    L->stats_launches = 0;
    int32_t *ctrl = reinterpret_cast<int32_t *>(ws + p.o_ctrl);
    MOE_LAUNCH(cudaMemsetAsync(ctrl, 0, p.ctrl_bytes, s));
    if (T == 0) return MOE_OK;
    MOE_MARK(L, 0, s);

    const int E = c.num_experts, k = c.num_active, S = c.num_shared;
    const moe_routing_t *rt = routing;
    float *logits = rt && rt->logits ? rt->logits : reinterpret_cast<float *>(ws + p.o_logits);
    int32_t *idx = rt && rt->topk_idx ? rt->topk_idx : reinterpret_cast<int32_t *>(ws + p.o_idx);
    float *gates = rt && rt->gates ? rt->gates : reinterpret_cast<float *>(ws + p.o_gates);
    int32_t *slot = rt && rt->slot ? rt->slot : reinterpret_cast<int32_t *>(ws + p.o_slot);
    L->fx = x;
    L->fgates = gates;
    int *nl = &L->fwd_launches;
    uint32_t *status = reinterpret_cast<uint32_t *>(ctrl + kCtrlStatus);

    RouterArgs ra;
    ra.x = x;
    ra.x_bf16 = 0;
    ra.w_gate = L->w.w_gate;
    ra.b_gate = L->w.b_gate;
    ra.noise = c.top_k_method == MOE_TOPK_NOISY ? logit_noise : nullptr;
    ra.sel_bias = c.use_selection_bias ? L->w.sel_bias : nullptr;
    ra.T = T;
    ra.d = c.input_dim;
    ra.E = E;
    ra.k = k;
    ra.logits = logits;
    ra.idx = idx;
    ra.gates = gates;
    ra.lse = reinterpret_cast<float *>(ws + p.o_lse);
    ra.psum_part = reinterpret_cast<float *>(ws + p.o_psum);
    ra.x_relu = 0;
    ra.logits_only = 0;
    // The tensor-core router (bf16 x): W_g, or the MLP gate's hidden matrix,
    // split into bf16 planes, then one fused kernel.
    auto fused = [&](const float *w, const float *b, int rows, float *out_logits, int route) -> int {
        const int E_pad = router_fused_epad(rows), BN = router_fused_bn(rows);
        __nv_bfloat16 *w_split = reinterpret_cast<__nv_bfloat16 *>(ws + p.o_wsplit);
        if (L->planes)  // split once by moe_prepare_router
            w_split = static_cast<__nv_bfloat16 *>(L->planes);
        else
            MOE_LAUNCH(launch_router_split(w, rows, E_pad, c.input_dim, w_split, L->num_sms, s, nl));
        CUtensorMap m_xr, m_ws;
        if (!encode_bf16_2d(&m_xr, x, c.input_dim, T, kBM) ||
            !encode_bf16_2d(&m_ws, w_split, 3ull * c.input_dim, E_pad, BN / 2))
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the router operands");
        RouterFusedArgs fa;
        fa.b_gate = b;
        fa.noise = route ? ra.noise : nullptr;
        fa.sel_bias = route ? ra.sel_bias : nullptr;
        fa.T = T;
        fa.d = c.input_dim;
        fa.E = rows;
        fa.k = k;
        fa.BN = BN;
        fa.n_tiles = E_pad / BN;
        fa.ksplit = p.ksplit;
        fa.n_mtiles = p.n_mtiles;
        fa.route = route;
        fa.logits = out_logits;
        fa.idx = idx;
        fa.gates = gates;
        fa.lse = ra.lse;
        fa.psum_part = ra.psum_part;
        fa.part = reinterpret_cast<float *>(ws + p.o_lpart);
        fa.counters = reinterpret_cast<int32_t *>(ws + p.o_rcnt);
        fa.status = status;
        fa.num_pairs = L->router_pairs;
        if (L->selftest_router_skip >= 0) {  // the timeout self-test
            fa.skip_stage = L->selftest_router_skip;
            fa.wait_limit_ns = kSelftestWaitNs;
        }
        MOE_LAUNCH(launch_router_fused(m_xr, m_ws, fa, s, nl));
        return MOE_OK;
    };
    if (c.use_mlp_gater) {
        // Hidden layer z = W_1 x + b_1 (pre-activations, [T][H] fp32), then the
        // output layer h = W_2 relu(z) + b_2 and the routing in one kernel.
        const int H = c.gater_hidden_dim;
        float *z = reinterpret_cast<float *>(ws + p.o_gz);
        if (L->tc) {
            const int rc = fused(L->w.gater_w1, L->w.gater_b1, H, z, 0);
            if (rc != MOE_OK) return rc;
        } else {
            RouterArgs rh = ra;
            rh.w_gate = L->w.gater_w1;
            rh.b_gate = L->w.gater_b1;
            rh.E = H;
            rh.logits = z;
            rh.logits_only = 1;
            rh.noise = nullptr;
            rh.sel_bias = nullptr;
            MOE_LAUNCH(launch_router(rh, s, nl));
        }
        ra.x = z;
        ra.x_bf16 = 0;
        ra.x_relu = 1;
        ra.d = H;
        MOE_LAUNCH(launch_router(ra, s, nl));
    } else if (L->tc) {
        const int rc = fused(L->w.w_gate, L->w.b_gate, E, logits, 1);
        if (rc != MOE_OK) return rc;
    } else {
        MOE_LAUNCH(launch_router(ra, s, nl));
    }
    MOE_MARK(L, 1, s);
    if (router_only) return MOE_OK;

    DispatchArgs da;
    da.idx = idx;
    da.T = T;
    da.rank_major = c.capacity_priority == MOE_PRIORITY_RANK ? 1 : 0;
    da.n_items = da.rank_major ? k * T : T;
    da.E = E;
    da.k = k;
    da.S = S;
    da.C = p.C;
    da.T_pad = p.T_pad;
    da.n_chunks = p.n_chunks;
    da.chunk_count = reinterpret_cast<int32_t *>(ws + p.o_ccount);
    da.chunk_base = reinterpret_cast<int32_t *>(ws + p.o_cbase);
    da.count_pre = reinterpret_cast<int32_t *>(ws + p.o_cpre);
    da.count_kept = reinterpret_cast<int32_t *>(ws + p.o_ckept);
    da.user_count_pre = rt ? rt->count_pre : nullptr;
    da.user_count_kept = rt ? rt->count_kept : nullptr;
    da.group_start = reinterpret_cast<int32_t *>(ws + p.o_gstart);
    da.group_rows = reinterpret_cast<int32_t *>(ws + p.o_grows);
    da.block_group = reinterpret_cast<int32_t *>(ws + p.o_bgroup);
    da.tok_tiles = reinterpret_cast<int4 *>(ws + p.o_toktiles);
    da.narrow_tiles = narrow_gemm(L, T) ? reinterpret_cast<int4 *>(ws + p.o_narrowtiles) : nullptr;
    da.tile_done = reinterpret_cast<int32_t *>(ws + p.o_tiledone);
    da.n_tile_done = p.n_tile_done;
    da.ctrl = ctrl;
    da.slot = slot;
    da.row_of = reinterpret_cast<int32_t *>(ws + p.o_rowof);
    da.row_assign = reinterpret_cast<int32_t *>(ws + p.o_rowassign);
    da.gates = gates;
    da.pre_start = reinterpret_cast<int32_t *>(ws + p.o_prestart);
    da.gate_sorted = reinterpret_cast<float *>(ws + p.o_gsorted);
    MOE_LAUNCH(launch_dispatch(da, s, nl));
    MOE_MARK(L, 2, s);

    if (L->tc) {
        ScatterArgs sa;
        sa.x = x;
        sa.xp = ws + p.o_xp;
        sa.row_of = da.row_of;
        sa.T = T;
        sa.k = k;
        sa.row_bytes = c.input_dim * 2;
        MOE_LAUNCH(launch_scatter(sa, L->num_sms, s, nl));
    }
    MOE_MARK(L, 3, s);
    return MOE_OK;
}

// Expert GEMMs over the forward's row space: every group, or (EP) only the
// shared experts' groups.
int fwd_expert_gemms(moe_layer_t *L, cudaStream_t s, bool shared_only) {
    const moe_config_t &c = L->cfg;
    const Plan &p = L->plan;
    char *ws = L->ws;
    const void *x = L->fx;
    const int T = p.T, E = c.num_experts, k = c.num_active, S = c.num_shared;
    if (T == 0 || (shared_only && S == 0)) return MOE_OK;
    int *nl = &L->fwd_launches;
    int32_t *ctrl = reinterpret_cast<int32_t *>(ws + p.o_ctrl);
    uint32_t *status = reinterpret_cast<uint32_t *>(ctrl + kCtrlStatus);
    DispatchArgs da;
    da.tok_tiles = reinterpret_cast<int4 *>(ws + p.o_toktiles);
    da.group_start = reinterpret_cast<int32_t *>(ws + p.o_gstart);
    da.group_rows = reinterpret_cast<int32_t *>(ws + p.o_grows);
    da.block_group = reinterpret_cast<int32_t *>(ws + p.o_bgroup);
    da.row_assign = reinterpret_cast<int32_t *>(ws + p.o_rowassign);

    if (L->tc) {
        PairGemmArgs g1;
        g1.tok_tiles = da.tok_tiles;
        g1.group_start = da.group_start;
        g1.ctrl = ctrl;
        g1.max_tok_tiles = p.max_tok_tiles;
        g1.N = c.expert_dim;
        g1.K = c.input_dim;
        g1.n_ftiles = gemm_pair_ftiles(c.expert_dim);
        g1.E = E;
        g1.w_shared_base = L->E_weights;
        if (shared_only) {  // the shared experts' tiles follow the routed ones
            g1.tile_base_word = kCtrlRoutedTiles;
            g1.fixed_tiles = S * ((p.T_pad + kTokTile - 1) / kTokTile);
        }
        if (!shared_only && narrow_gemm(L, T)) {
            g1.tok_tiles = reinterpret_cast<const int4 *>(ws + p.o_narrowtiles);
            g1.tiles_count_word = kCtrlNumNarrowTiles;
            g1.max_tok_tiles = p.max_narrow_tiles;
            g1.narrow = 1;
        }
        g1.use_s = 1;
        g1.half_last = !g1.narrow && gemm_pair_half_last(c.expert_dim);
        g1.out = reinterpret_cast<__nv_bfloat16 *>(ws + p.o_h);
        g1.bias = L->w.b1;
        g1.act = c.activation;
        g1.status = status;
        g1.work_counter = ctrl + kCtrlWork1;
        g1.num_pairs = L->num_pairs;
        PairGemmArgs g2 = g1;
        if (L->selftest_skip_stage >= 0) {  // the timeout self-test: GEMM 1 misses one stage's loads
            g1.skip_stage = L->selftest_skip_stage;
            g1.wait_limit_ns = kSelftestWaitNs;
        }
        g2.N = c.output_dim;
        g2.K = c.expert_dim;
        g2.n_ftiles = gemm_pair_ftiles(c.output_dim);
        g2.use_s = 0;
        g2.half_last = !g2.narrow && gemm_pair_half_last(c.output_dim);
        g2.out = reinterpret_cast<__nv_bfloat16 *>(ws + p.o_o);
        g2.bias = L->w.b2;
        g2.act = -1;
        g2.work_counter = ctrl + kCtrlWork2;
        PairMaps m1, m2;
        m1.w = L->map_w1;
        m1.wh = L->map_w1h;
        m2.w = L->map_w2;
        m2.wh = L->map_w2h;
        if (!encode_bf16_2d(&m1.t, ws + p.o_xp, c.input_dim, p.R_routed_max, 128) ||
            !encode_bf16_2d(&m1.t16, ws + p.o_xp, c.input_dim, p.R_routed_max, 16) ||
            !encode_bf16_2d(&m1.s, x, c.input_dim, T, 128) || !encode_bf16_2d(&m1.s16, x, c.input_dim, T, 16) ||
            !encode_bf16_2d(&m2.t, ws + p.o_h, c.expert_dim, p.R_max, 128) ||
            !encode_bf16_2d(&m2.t16, ws + p.o_h, c.expert_dim, p.R_max, 16) ||
            !encode_bf16_store(&m1.out, ws + p.o_h, c.expert_dim, p.R_max) ||
            !encode_bf16_store(&m2.out, ws + p.o_o, c.output_dim, p.R_max))
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the activations");
        m2.s = m2.t;
        m2.s16 = m2.t16;
        if (!shared_only) {
            // Both layers in one launch: layer 2's units of a token tile start
            // as soon as its layer-1 units have stored H, so layer 2 fills
            // layer 1's last wave (3% off the decode step, where the two
            // layers stream weights from HBM; a few tenths of a percent at
            // e64). The stage events of the two GEMMs then both follow this
            // launch.
            g1.tile_done = reinterpret_cast<int32_t *>(ws + p.o_tiledone);
            MOE_LAUNCH(launch_gemm_pair(m1, g1, &m2, &g2, s, nl));
            MOE_MARK(L, 4, s);
        } else {
            MOE_LAUNCH(launch_gemm_pair(m1, g1, nullptr, nullptr, s, nl));
            MOE_MARK(L, 4, s);
            MOE_LAUNCH(launch_gemm_pair(m2, g2, nullptr, nullptr, s, nl));
        }
        MOE_MARK(L, 5, s);
    } else {
        GemmSimtArgs s1;
        s1.block_group = da.block_group;
        s1.group_start = da.group_start;
        s1.group_rows = da.group_rows;
        s1.ctrl = ctrl;
        s1.max_row_blocks = p.max_row_blocks;
        s1.N = c.expert_dim;
        s1.K = c.input_dim;
        s1.E = E;
        s1.k = k;
        s1.row_assign = da.row_assign;
        s1.bias = L->w.b1;
        s1.out = reinterpret_cast<float *>(ws + p.o_h);
        s1.act = c.activation;
        s1.a = static_cast<const float *>(x);
        s1.gather = 1;
        s1.w = static_cast<const float *>(L->w.w1);
        MOE_LAUNCH(launch_gemm_simt(s1, s, nl));
        MOE_MARK(L, 4, s);
        GemmSimtArgs s2 = s1;
        s2.N = c.output_dim;
        s2.K = c.expert_dim;
        s2.bias = L->w.b2;
        s2.out = reinterpret_cast<float *>(ws + p.o_o);
        s2.act = -1;
        s2.a = reinterpret_cast<const float *>(ws + p.o_h);
        s2.gather = 0;
        s2.w = static_cast<const float *>(L->w.w2);
        MOE_LAUNCH(launch_gemm_simt(s2, s, nl));
        MOE_MARK(L, 5, s);
    }

    return MOE_OK;
}

// Credit norms (hidden reading) and the combine of the forward's outputs.
int fwd_combine(moe_layer_t *L, void *y, cudaStream_t s) {
    const moe_config_t &c = L->cfg;
    const Plan &p = L->plan;
    char *ws = L->ws;
    const int T = p.T, E = c.num_experts, k = c.num_active, S = c.num_shared;
    if (T == 0) return MOE_OK;
    int *nl = &L->fwd_launches;
    int32_t *ctrl = reinterpret_cast<int32_t *>(ws + p.o_ctrl);
    DispatchArgs da;
    da.row_of = reinterpret_cast<int32_t *>(ws + p.o_rowof);
    da.row_assign = reinterpret_cast<int32_t *>(ws + p.o_rowassign);
    da.group_start = reinterpret_cast<int32_t *>(ws + p.o_gstart);
    float *gates = L->fgates;
    float *row_norm2 = nullptr;
    if (c.credit_norm == MOE_CREDIT_HIDDEN) {
        RowNormArgs rn;
        rn.m = ws + p.o_h;
        rn.n = c.expert_dim;
        rn.bf16 = L->tc ? 1 : 0;
        rn.row_assign = da.row_assign;
        rn.ctrl = ctrl;
        rn.max_rows = p.R_routed_max;
        rn.norm2 = row_norm2 = reinterpret_cast<float *>(ws + p.o_rownorm);
        MOE_LAUNCH(launch_row_norms(rn, L->num_sms, s, nl));
    }

    CombineArgs ca;
    ca.o = ws + p.o_o;
    ca.row_norm2 = row_norm2;
    ca.row_of = da.row_of;
    ca.gates = gates;
    ca.group_start = da.group_start;
    ca.T = T;
    ca.O = c.output_dim;
    ca.E = E;
    ca.S = S;
    ca.k = k;
    ca.bf16 = c.dtype == MOE_DTYPE_BF16;
    ca.y = y;
    ca.credit = reinterpret_cast<float *>(ws + p.o_credit);
    MOE_LAUNCH(launch_combine(ca, L->num_sms, s, nl));
    MOE_MARK(L, 6, s);
    return MOE_OK;
}

}  // namespace

extern "C" {

int moe_forward(moe_layer_t *L, const void *x, int32_t T, const float *logit_noise, void *workspace, size_t ws_bytes,
                void *y, const moe_routing_t *routing, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (L->cfg.ep_size > 1)
        return fail(MOE_ERR_STATE, "an expert-parallel layer runs moe_ep_dispatch / moe_ep_experts / moe_ep_combine");
    if (T > 0 && !y) return fail(MOE_ERR_INVALID_ARG, "y is required when T > 0");
    if (reinterpret_cast<uintptr_t>(y) % 16) return fail(MOE_ERR_INVALID_ARG, "y must be 16-byte aligned");
    cudaStream_t s = as_stream(stream_v);
    int rc = fwd_route(L, x, T, logit_noise, workspace, ws_bytes, routing, s);
    if (rc != MOE_OK || T == 0) return rc;
    rc = fwd_expert_gemms(L, s, false);
    if (rc != MOE_OK) return rc;
    return fwd_combine(L, y, s);
}

// ------------------------------------------------------------ expert parallelism

int moe_ep_dispatch(moe_layer_t *L, const void *x, int32_t T, const float *logit_noise, void *workspace,
                    size_t ws_bytes, const moe_routing_t *routing, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (L->cfg.ep_size < 2) return fail(MOE_ERR_STATE, "moe_ep_* calls are for layers with ep_size > 1");
    return fwd_route(L, x, T, logit_noise, workspace, ws_bytes, routing, as_stream(stream_v));
}

int moe_ep_layout(moe_layer_t *L, int32_t *expert_rows, void **rows_in, void **rows_out, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!expert_rows) return fail(MOE_ERR_INVALID_ARG, "expert_rows is NULL");
    if (!L->has_forward) return fail(MOE_ERR_STATE, "moe_ep_layout before moe_ep_dispatch");
    const int E = L->cfg.num_experts;
    const Plan &p = L->plan;
    if (rows_in) *rows_in = L->ws + p.o_xp;
    if (rows_out) *rows_out = L->ws + p.o_o;
    if (p.T == 0) {
        std::memset(expert_rows, 0, sizeof(int32_t) * E);
        return MOE_OK;
    }
    std::vector<int32_t> gs(E + 1);
    cudaStream_t s = as_stream(stream_v);
    MOE_LAUNCH(cudaMemcpyAsync(gs.data(), L->ws + p.o_gstart, sizeof(int32_t) * (E + 1), cudaMemcpyDeviceToHost, s));
    MOE_LAUNCH(cudaStreamSynchronize(s));
    for (int e = 0; e < E; ++e) expert_rows[e] = gs[e + 1] - gs[e];
    return MOE_OK;
}

namespace {
struct EpPlan {
    size_t o_ctrl, o_tiles, o_h, total;
    int max_tiles;
};
EpPlan ep_plan(const moe_layer &L, int R) {
    EpPlan q;
    const int E = L.cfg.num_experts;
    q.max_tiles = std::max(1, std::min(R / kTokTile + E, R / kRowBlock));
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    q.o_ctrl = take(kCtrlWords * 4);
    q.o_tiles = take((size_t)q.max_tiles * 16);
    q.o_h = take((size_t)R * L.cfg.expert_dim * 2);
    q.total = off;
    return q;
}
}  // namespace

size_t moe_ep_experts_workspace_bytes(const moe_layer_t *L, int32_t R) {
    if (!L || R < 0) return 0;
    return ep_plan(*L, R).total;
}

int moe_ep_experts(moe_layer_t *L, const void *recv_x, const int32_t *recv_rows, int32_t R, void *recv_out,
                   void *workspace, size_t ws_bytes, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    const moe_config_t &c = L->cfg;
    if (c.ep_size < 2) return fail(MOE_ERR_STATE, "moe_ep_* calls are for layers with ep_size > 1");
    if (R < 0) return fail(MOE_ERR_INVALID_ARG, "R must be >= 0");
    if (R % kRowBlock) return fail(MOE_ERR_INVALID_ARG, "R must be a multiple of %d (got %d)", kRowBlock, R);
    if (R == 0) return MOE_OK;
    if (!recv_x || !recv_rows || !recv_out || !workspace)
        return fail(MOE_ERR_INVALID_ARG, "recv_x, recv_rows, recv_out and workspace are required");
    const EpPlan q = ep_plan(*L, R);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (ws_bytes < q.total) return fail(MOE_ERR_WORKSPACE, "workspace too small: %zu given, %zu needed", ws_bytes, q.total);
    if ((reinterpret_cast<uintptr_t>(recv_x) | reinterpret_cast<uintptr_t>(recv_out)) % 16)
        return fail(MOE_ERR_INVALID_ARG, "recv_x and recv_out must be 16-byte aligned");
    cudaStream_t s = as_stream(stream_v);
    char *ws = static_cast<char *>(workspace);
    int32_t *ctrl = reinterpret_cast<int32_t *>(ws + q.o_ctrl);
    int4 *tiles = reinterpret_cast<int4 *>(ws + q.o_tiles);
    int launches = 0;
    EpTilesArgs ta;
    ta.recv_rows = recv_rows;
    ta.G = c.ep_size;
    ta.El = L->E_weights;
    ta.R = R;
    ta.tiles = tiles;
    ta.ctrl = ctrl;
    MOE_LAUNCH(launch_ep_tiles(ta, s, &launches));

    PairGemmArgs g1;
    g1.tok_tiles = tiles;
    g1.group_start = nullptr;
    g1.ctrl = ctrl;
    g1.max_tok_tiles = q.max_tiles;
    g1.N = c.expert_dim;
    g1.K = c.input_dim;
    g1.n_ftiles = gemm_pair_ftiles(c.expert_dim);
    g1.E = L->E_weights;  // every received group is a routed expert held here
    g1.w_shared_base = L->E_weights;
    g1.use_s = 0;
    g1.half_last = gemm_pair_half_last(c.expert_dim);
    g1.out = reinterpret_cast<__nv_bfloat16 *>(ws + q.o_h);
    g1.bias = L->w.b1;
    g1.act = c.activation;
    g1.status = reinterpret_cast<uint32_t *>(ctrl + kCtrlStatus);
    g1.work_counter = ctrl + kCtrlWork1;
    g1.num_pairs = L->num_pairs;
    PairGemmArgs g2 = g1;
    g2.N = c.output_dim;
    g2.K = c.expert_dim;
    g2.n_ftiles = gemm_pair_ftiles(c.output_dim);
    g2.half_last = gemm_pair_half_last(c.output_dim);
    g2.out = reinterpret_cast<__nv_bfloat16 *>(recv_out);
    g2.bias = L->w.b2;
    g2.act = -1;
    g2.work_counter = ctrl + kCtrlWork2;
    PairMaps m1, m2;
    m1.w = L->map_w1;
    m1.wh = L->map_w1h;
    m2.w = L->map_w2;
    m2.wh = L->map_w2h;
    if (!encode_bf16_2d(&m1.t, recv_x, c.input_dim, R, 128) || !encode_bf16_2d(&m1.t16, recv_x, c.input_dim, R, 16) ||
        !encode_bf16_2d(&m2.t, ws + q.o_h, c.expert_dim, R, 128) ||
        !encode_bf16_2d(&m2.t16, ws + q.o_h, c.expert_dim, R, 16) ||
        !encode_bf16_store(&m1.out, ws + q.o_h, c.expert_dim, R) || !encode_bf16_store(&m2.out, recv_out, c.output_dim, R))
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the received rows");
    m1.s = m1.t;
    m1.s16 = m1.t16;
    m2.s = m2.t;
    m2.s16 = m2.t16;
    MOE_LAUNCH(launch_gemm_pair(m1, g1, nullptr, nullptr, s, &launches));
    MOE_LAUNCH(launch_gemm_pair(m2, g2, nullptr, nullptr, s, &launches));
    return MOE_OK;
}

int moe_ep_combine(moe_layer_t *L, void *y, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (L->cfg.ep_size < 2) return fail(MOE_ERR_STATE, "moe_ep_* calls are for layers with ep_size > 1");
    if (!L->has_forward) return fail(MOE_ERR_STATE, "moe_ep_combine before moe_ep_dispatch");
    if (L->plan.T > 0 && !y) return fail(MOE_ERR_INVALID_ARG, "y is required when T > 0");
    if (reinterpret_cast<uintptr_t>(y) % 16) return fail(MOE_ERR_INVALID_ARG, "y must be 16-byte aligned");
    cudaStream_t s = as_stream(stream_v);
    int rc = fwd_expert_gemms(L, s, true);
    if (rc != MOE_OK) return rc;
    return fwd_combine(L, y, s);
}

}  // extern "C"

namespace {

// Enqueues the partial sums of the most recent forward into `partials` (and,
// with fin, the statistics from them in the same launch).
int enqueue_partials(moe_layer_t *L, const float *token_loss, float *partials, cudaStream_t s, int *launches,
                     const FinalizeArgs *fin = nullptr) {
    const Plan &p = L->plan;
    const moe_config_t &c = L->cfg;
    char *ws = L->ws;
    StatsArgs sa;
    sa.psum_part = reinterpret_cast<const float *>(ws + p.o_psum);
    sa.n_chunks = p.n_stat_chunks;
    sa.lse = reinterpret_cast<const float *>(ws + p.o_lse);
    sa.count_pre = reinterpret_cast<const int32_t *>(ws + p.o_cpre);
    sa.group_start = reinterpret_cast<const int32_t *>(ws + p.o_gstart);
    sa.group_rows = reinterpret_cast<const int32_t *>(ws + p.o_grows);
    sa.row_assign = reinterpret_cast<const int32_t *>(ws + p.o_rowassign);
    sa.credit = reinterpret_cast<const float *>(ws + p.o_credit);
    sa.token_loss = token_loss;
    sa.ctrl = reinterpret_cast<const int32_t *>(ws + p.o_ctrl);
    sa.pre_start = reinterpret_cast<const int32_t *>(ws + p.o_prestart);
    sa.gate_sorted = reinterpret_cast<const float *>(ws + p.o_gsorted);
    sa.T = p.T;
    sa.E = c.num_experts;
    sa.k = c.num_active;
    sa.partials = partials;
    sa.done_counter = reinterpret_cast<int32_t *>(ws + p.o_ctrl) + kCtrlStatsDone;
    MOE_LAUNCH(launch_stat_partials(sa, fin, s, launches));
    return MOE_OK;
}

FinalizeArgs finalize_args(const moe_layer_t *L, const float *partials, bool has_loss, const moe_stats_t *out) {
    const moe_config_t &c = L->cfg;
    FinalizeArgs fa;
    fa.partials = partials;
    fa.E = c.num_experts;
    fa.k = c.num_active;
    fa.alpha = c.load_balance_coef;
    fa.beta = c.z_loss_coef;
    fa.f = out->f;
    fa.p_mean = out->p_mean;
    fa.l_aux = out->l_aux;
    fa.l_z = out->l_z;
    fa.expert_loss = has_loss ? out->expert_loss : nullptr;
    fa.n_dropped = out->n_dropped;
    fa.importance = out->importance;
    fa.cv_load = out->cv_load;
    fa.cv_importance = out->cv_importance;
    fa.l_total = out->l_total;
    return fa;
}

int enqueue_finalize(moe_layer_t *L, const float *partials, bool has_loss, const moe_stats_t *out, cudaStream_t s,
                     int *launches) {
    const FinalizeArgs fa = finalize_args(L, partials, has_loss, out);
    MOE_LAUNCH(launch_stats_finalize(fa, s, launches));
    return MOE_OK;
}

}  // namespace

extern "C" {

int moe_aux_stats(moe_layer_t *L, const float *token_loss, const moe_stats_t *out, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    if (!L->has_forward) return fail(MOE_ERR_STATE, "moe_aux_stats called before any moe_forward");
    const Plan &p = L->plan;
    const moe_config_t &c = L->cfg;
    cudaStream_t s = as_stream(stream_v);
    L->stats_launches = 0;
    if (p.T == 0) return MOE_OK;
    float *partials = reinterpret_cast<float *>(L->ws + p.o_partials);
    const FinalizeArgs fin = finalize_args(L, partials, token_loss != nullptr, out);
    int rc = enqueue_partials(L, token_loss, partials, s, &L->stats_launches, &fin);
    if (rc != MOE_OK) return rc;
    if (out->credit)
        MOE_LAUNCH(cudaMemcpyAsync(out->credit, L->ws + p.o_credit, (size_t)p.T * c.num_active * 4,
                                   cudaMemcpyDeviceToDevice, s));
    MOE_MARK(L, 7, s);
    return MOE_OK;
}

int moe_stat_partials(moe_layer_t *L, const float *token_loss, float *partials, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!partials) return fail(MOE_ERR_INVALID_ARG, "partials is NULL");
    if (!L->has_forward) return fail(MOE_ERR_STATE, "moe_stat_partials called before any moe_forward");
    cudaStream_t s = as_stream(stream_v);
    if (L->plan.T == 0) {
        MOE_LAUNCH(cudaMemsetAsync(partials, 0, (size_t)(4 * L->cfg.num_experts + 3) * 4, s));
        return MOE_OK;
    }
    int launches = 0;
    return enqueue_partials(L, token_loss, partials, s, &launches);
}

int moe_stats_from_partials(moe_layer_t *L, const float *partials, int32_t has_token_loss, const moe_stats_t *out,
                            void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!partials) return fail(MOE_ERR_INVALID_ARG, "partials is NULL");
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    int launches = 0;
    return enqueue_finalize(L, partials, has_token_loss != 0, out, as_stream(stream_v), &launches);
}

int moe_update_selection_bias(moe_layer_t *L, const float *partials, float gamma, float *sel_bias, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!sel_bias) return fail(MOE_ERR_INVALID_ARG, "sel_bias is NULL");
    if (gamma != gamma) return fail(MOE_ERR_INVALID_ARG, "gamma is NaN");
    if (!partials && !L->has_forward)
        return fail(MOE_ERR_STATE, "moe_update_selection_bias without partials needs a previous moe_forward");
    BiasUpdateArgs ba;
    ba.partials = partials;
    ba.count_pre = partials ? nullptr : reinterpret_cast<const int32_t *>(L->ws + L->plan.o_cpre);
    ba.T = partials ? 0 : L->plan.T;
    ba.E = L->cfg.num_experts;
    ba.k = L->cfg.num_active;
    ba.gamma = gamma;
    ba.sel_bias = sel_bias;
    if (!partials && ba.T == 0) return MOE_OK;
    int launches = 0;
    MOE_LAUNCH(launch_bias_update(ba, as_stream(stream_v), &launches));
    return MOE_OK;
}

int moe_dro_update(moe_layer_t *L, const float *expert_loss, float ema, float eta, float *lhat, float *mu,
                   float *objective, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!expert_loss || !lhat || !mu) return fail(MOE_ERR_INVALID_ARG, "expert_loss, lhat and mu are required");
    if (!std::isfinite(ema) || !std::isfinite(eta)) return fail(MOE_ERR_INVALID_ARG, "ema and eta must be finite");
    DroArgs da;
    da.l = expert_loss;
    da.lhat = lhat;
    da.mu = mu;
    da.objective = objective;
    da.E = L->cfg.num_experts;
    da.ema = ema;
    da.eta = eta;
    int launches = 0;
    MOE_LAUNCH(launch_dro_update(da, as_stream(stream_v), &launches));
    return MOE_OK;
}

size_t moe_router_planes_bytes(const moe_layer_t *L) {
    if (!L || !L->tc) return 0;
    const int rows = L->cfg.use_mlp_gater ? L->cfg.gater_hidden_dim : L->cfg.num_experts;
    return (size_t)router_fused_epad(rows) * 3 * L->cfg.input_dim * 2;
}

int moe_prepare_router(moe_layer_t *L, void *planes, size_t bytes, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!L->tc) return fail(MOE_ERR_UNSUPPORTED, "fp32 layers route on CUDA cores from the fp32 router matrix");
    if (!planes) {
        L->planes = nullptr;
        return MOE_OK;
    }
    const size_t need = moe_router_planes_bytes(L);
    if (bytes < need) return fail(MOE_ERR_WORKSPACE, "router planes: %zu bytes given, %zu needed", bytes, need);
    if (reinterpret_cast<uintptr_t>(planes) % 256) return fail(MOE_ERR_WORKSPACE, "planes must be 256-byte aligned");
    const moe_config_t &c = L->cfg;
    const int rows = c.use_mlp_gater ? c.gater_hidden_dim : c.num_experts;
    const float *w = c.use_mlp_gater ? L->w.gater_w1 : L->w.w_gate;
    int launches = 0;
    MOE_LAUNCH(launch_router_split(w, rows, router_fused_epad(rows), c.input_dim, static_cast<__nv_bfloat16 *>(planes),
                                   L->num_sms, as_stream(stream_v), &launches));
    L->planes = planes;
    return MOE_OK;
}

int moe_selftest_gemm_timeout(moe_layer_t *L, const void *x, int32_t T, void *workspace, size_t ws_bytes, void *y,
                              void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!L->tc || L->cfg.ep_size > 1)
        return fail(MOE_ERR_UNSUPPORTED, "the self-test runs the tensor-core expert GEMM of a bf16 layer, ep_size 1");
    if (L->cfg.top_k_method != MOE_TOPK_GREEDY) return fail(MOE_ERR_UNSUPPORTED, "the self-test needs GREEDY top-k");
    if (T <= 0) return fail(MOE_ERR_INVALID_ARG, "the self-test needs T > 0");
    if (L->cfg.input_dim < 3 * kBK)
        return fail(MOE_ERR_UNSUPPORTED, "the self-test needs input_dim >= %d (three K stages)", 3 * kBK);
    L->selftest_skip_stage = 2;
    int rc = moe_forward(L, x, T, nullptr, workspace, ws_bytes, y, nullptr, stream_v);
    L->selftest_skip_stage = -1;
    if (rc != MOE_OK) return rc;
    cudaStream_t s = as_stream(stream_v);
    MOE_LAUNCH(cudaStreamSynchronize(s));
    uint32_t st = 0;
    MOE_LAUNCH(cudaMemcpy(&st, L->ws + L->plan.o_ctrl + kCtrlStatus * 4, 4, cudaMemcpyDeviceToHost));
    if (!(st & kDevTimeout)) return fail(MOE_ERR_INTERNAL, "expert GEMM 1 missed a stage but reported no timeout");
    return MOE_OK;
}

int moe_selftest_router_timeout(moe_layer_t *L, const void *x, int32_t T, void *workspace, size_t ws_bytes,
                                void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!L->tc || L->cfg.use_mlp_gater)
        return fail(MOE_ERR_UNSUPPORTED, "the self-test runs the fused router of a bf16 layer with a linear router");
    if (L->cfg.top_k_method != MOE_TOPK_GREEDY) return fail(MOE_ERR_UNSUPPORTED, "the self-test needs GREEDY top-k");
    if (T <= 0) return fail(MOE_ERR_INVALID_ARG, "the self-test needs T > 0");
    if (L->cfg.input_dim < 3 * kBK)
        return fail(MOE_ERR_UNSUPPORTED, "the self-test needs input_dim >= %d (three K stages)", 3 * kBK);
    // The router alone: its outputs are incomplete after the timeout, so no
    // later kernel of the forward may read them.
    L->selftest_router_skip = 2;
    int rc = fwd_route(L, x, T, nullptr, workspace, ws_bytes, nullptr, as_stream(stream_v), true);
    L->selftest_router_skip = -1;
    if (rc != MOE_OK) return rc;
    L->has_forward = false;  // nothing for moe_aux_stats to read
    cudaStream_t s = as_stream(stream_v);
    MOE_LAUNCH(cudaStreamSynchronize(s));
    uint32_t st = 0;
    MOE_LAUNCH(cudaMemcpy(&st, L->ws + L->plan.o_ctrl + kCtrlStatus * 4, 4, cudaMemcpyDeviceToHost));
    if (!(st & kDevTimeout)) return fail(MOE_ERR_INTERNAL, "the router missed a stage but reported no timeout");
    return MOE_OK;
}

int moe_device_status(moe_layer_t *L, void *stream_v) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!L->has_forward) return fail(MOE_ERR_STATE, "no forward has run on this layer");
    cudaStream_t s = as_stream(stream_v);
    MOE_LAUNCH(cudaStreamSynchronize(s));
    uint32_t st = 0;
    MOE_LAUNCH(cudaMemcpy(&st, L->ws + L->plan.o_ctrl + kCtrlStatus * 4, 4, cudaMemcpyDeviceToHost));
    if (st & kDevTimeout) return fail(MOE_ERR_TIMEOUT, "a bounded device-side wait gave up (status 0x%x)", st);
    return MOE_OK;
}

int moe_set_timing_events(moe_layer_t *L, void *const *events) {
    g_last_error.clear();
    if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
    if (!events) {
        L->timing = false;
        return MOE_OK;
    }
    for (int i = 0; i < MOE_TIMING_EVENTS; ++i) {
        if (!events[i]) return fail(MOE_ERR_INVALID_ARG, "events[%d] is NULL", i);
        L->ev[i] = reinterpret_cast<cudaEvent_t>(events[i]);
    }
    L->timing = true;
    return MOE_OK;
}

int32_t moe_launch_count(const moe_layer_t *L) { return L ? L->fwd_launches + L->stats_launches : 0; }

void moe_destroy(moe_layer_t *L) { delete L; }

const char *moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
        case MOE_ERR_STATE: return "MOE_ERR_STATE";
        case MOE_ERR_INTERNAL: return "MOE_ERR_INTERNAL";
        default: return "MOE_ERR_UNKNOWN";
    }
}

const char *moe_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
