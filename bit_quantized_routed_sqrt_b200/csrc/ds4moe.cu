// ds4moe.cu -- host side of the C ABI declared in include/ds4moe.h.
//
// One handle = one layer on one device: its repacked weights, a workspace sized for
// max_tokens, and the launch logic of the two forward paths (batched GEMV for small T,
// grouped path for large T).  Everything runs on the caller's stream; nothing here
// computes on the host except weight norms at load time.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/ds4moe.h"
#include "common.cuh"
#include "decode.cuh"
#include "misc.cuh"
#include "repack.cuh"
#include "router.cuh"
#include "prefill.cuh"

using namespace ds4;

struct ds4moe {
    int device = 0;
    ds4moe_config cfg{};
    int num_sms = 148;
    cudaStream_t last_stream = nullptr;
    bool loaded = false;
    std::string err;
    // weights
    uint8_t *gate = nullptr, *up = nullptr, *down = nullptr;
    size_t gu_bytes = 0, d_bytes = 0;
    __nv_bfloat16 *wr = nullptr, *sg = nullptr, *su = nullptr, *sd = nullptr;
    float *bias = nullptr, *wr_norm = nullptr;
    bool has_bias = false;
    // workspace
    void *ws = nullptr;
    size_t ws_bytes = 0;
    double *logits = nullptr;
    float *labs = nullptr;
    RouteOut ro{};
    // batched-GEMV path (sized for min(max_tokens, MAX_DECODE_T) tokens)
    uint8_t *xrec = nullptr;     // int16 token records
    uint8_t *hrec = nullptr;   // decode: per (token, slot) pair, the routed h record
    float *hs = nullptr, *o = nullptr, *s = nullptr;
    DecCtl *ctl = nullptr;
    int *blk_cnt = nullptr;
    unsigned long long *blk_mask = nullptr;
    uint16_t *x_stage = nullptr;
    float *y_stage = nullptr;
    int *status = nullptr;
    int *dbg = nullptr;      // [8] first device-side check violation
    unsigned long long *fallbacks = nullptr;
    PrefillWork pw{};
    __half *sg16 = nullptr, *su16 = nullptr, *sd16 = nullptr;   // shared expert in fp16 (grouped path)
    CUtensorMap tm_x{}, tm_h{}, tm_sg{}, tm_su{}, tm_sd{}, tm_wr{};
    bool maps_ok = false;
    unsigned long long *trace = nullptr;
    int trace_units = 0;     // unit records of the trace buffer (then 2 per CTA, then 4)
    // profiling
    cudaEvent_t ev[9] = {};
    int n_ev = 0;
    int last_path = 0, last_T = 0;
    bool test_timeout_pending = false;   // DS4MOE_FLAG_TEST_TIMEOUT: the next batched-GEMV forward
};

namespace {

ds4moe_status fail(ds4moe *h, ds4moe_status st, const char *fmt, ...) {
    if (h) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        h->err = buf;
    }
    return st;
}

#define CK(h, call)                                                                                     \
    do {                                                                                                \
        cudaError_t e_ = (call);                                                                        \
        if (e_ != cudaSuccess)                                                                          \
            return fail((h), e_ == cudaErrorMemoryAllocation ? DS4MOE_ENOMEM : DS4MOE_ECUDA, "%s: %s (%s:%d)", \
                        #call, cudaGetErrorString(e_), __FILE__, __LINE__);                           \
    } while (0)

#define CKL(h)                                                                                          \
    do {                                                                                                \
        cudaError_t e_ = cudaGetLastError();                                                            \
        if (e_ != cudaSuccess)                                                                          \
            return fail((h), DS4MOE_ECUDA, "kernel launch: %s (%s:%d)", cudaGetErrorString(e_), __FILE__, __LINE__); \
    } while (0)

struct Carver {
    char *base;
    size_t off = 0;
    template <class T>
    T *take(size_t count) {
        off = (off + 255) & ~(size_t)255;
        T *p = reinterpret_cast<T *>(base ? base + off : nullptr);
        off += count * sizeof(T);
        return p;
    }
};

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Host-side fault injection (test hook): DS4MOE_FAULT=alloc makes ds4moe_create fail as if
// its workspace allocation had failed (before any CUDA call); =h2d makes
// ds4moe_load_q2k_experts fail at its first host-to-device copy; =launch makes the next
// forward or routing call fail before its first launch.  Nothing reaches the GPU.
bool injected(const char *what) {
    const char *v = getenv("DS4MOE_FAULT");
    return v && strcmp(v, what) == 0;
}

int npl_of(int E) { return E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8; }

void layout_workspace(ds4moe *h, Carver &c) {
    const ds4moe_config &g = h->cfg;
    const size_t Tm = g.max_tokens, P = Tm * g.top_k, E = g.n_experts, H = g.hidden, I = g.inter, Is = g.shared_inter;
    const size_t NB = (Tm + 63) / 64;
    h->logits = c.take<double>(Tm * E);
    h->labs = c.take<float>(Tm * E);
    h->ro.topk_idx = c.take<int>(P);
    h->ro.topk_w = c.take<float>(P);
    h->ro.offsets = c.take<int>(E + 1);
    h->ro.sorted_token = c.take<int>(P);
    h->ro.sorted_slot = c.take<int>(P);
    h->ro.inv_pos = c.take<int>(P);
    h->ro.active = c.take<int>(E);
    h->ro.n_active = c.take<int>(1);
    const size_t Td = std::min<size_t>(Tm, MAX_DECODE_T), Pd = Td * g.top_k;
    h->xrec = c.take<uint8_t>(Td * (size_t)make_dec_plan(1, (int)H, (int)E, g.top_k, (int)I, (int)Is).xrec);
    h->hs = c.take<float>(Td * (Is ? Is : 1));
    h->hrec = c.take<uint8_t>(Pd * (size_t)make_dec_plan(1, (int)H, (int)E, g.top_k, (int)I, (int)Is).hrec);
    h->o = c.take<float>(Pd * H);
    h->s = c.take<float>(Td * H);
    h->ctl = c.take<DecCtl>(1);
    h->blk_cnt = c.take<int>(NB * E);
    h->blk_mask = c.take<unsigned long long>(NB * E);
    h->x_stage = c.take<uint16_t>(Tm * H);
    h->y_stage = c.take<float>(Tm * H);
    h->status = c.take<int>(1);
    h->dbg = c.take<int>(8);
    h->fallbacks = c.take<unsigned long long>(1);
    prefill_layout(h->pw, c, g.max_tokens, g.top_k, g.n_experts, g.hidden, g.inter, g.shared_inter);
}

void free_weights(ds4moe *h) {
    for (void *p : {(void *)h->gate, (void *)h->up, (void *)h->down, (void *)h->wr, (void *)h->sg, (void *)h->su,
                    (void *)h->sd, (void *)h->bias, (void *)h->wr_norm, (void *)h->sg16, (void *)h->su16,
                    (void *)h->sd16})
        if (p) cudaFree(p);
    h->sg16 = h->su16 = h->sd16 = nullptr;
    h->maps_ok = false;
    h->gate = h->up = h->down = nullptr;
    h->wr = h->sg = h->su = h->sd = nullptr;
    h->bias = h->wr_norm = nullptr;
    h->loaded = false;
}

PFN_cuTensorMapEncodeTiled_v12000 tmap_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D 16-bit tensor map [rows][cols] (row-major, fp16 or bf16) with a {64, box_rows} box and
// 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_rows,
              CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT16) {
    auto enc = tmap_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)PF_BK, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Upper bound of the work units of one batched-GEMV launch of T tokens (trace sizing).
int decode_unit_bound(const ds4moe_config &g, int T) {
    const DecPlan pl = make_dec_plan(T, g.hidden, g.n_experts, g.top_k, g.inter, g.shared_inter);
    const int groups = std::min(T * g.top_k, g.n_experts * ((T + DK_TU - 1) / DK_TU));
    return pl.nSG + pl.nSD + groups * (pl.RGI + pl.RPH);
}

DecArgs decode_args(ds4moe *h, const void *x, int T, float *y, bool route_only) {
    DecArgs a{};
    const ds4moe_config &g = h->cfg;
    a.T = T; a.H = g.hidden; a.E = g.n_experts; a.k = g.top_k; a.I = g.inter; a.Is = g.shared_inter;
    a.pl = make_dec_plan(T, g.hidden, g.n_experts, g.top_k, g.inter, g.shared_inter);
    a.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    a.wr = h->wr; a.bias = h->has_bias ? h->bias : nullptr;
    a.sg = h->sg; a.su = h->su; a.sd = h->sd;
    a.gate = h->gate; a.up = h->up; a.down = h->down;
    a.gu_bytes = h->gu_bytes; a.d_bytes = h->d_bytes;
    a.logits = h->logits; a.labs = h->labs; a.ro = h->ro;
    a.xrec = h->xrec;
    a.hs = h->hs; a.hrec = h->hrec;
    a.o = h->o; a.s = h->s; a.y = y;
    a.ctl = h->ctl;
    a.status = h->status;
    a.route_only = route_only ? 1 : 0;
    a.test_timeout = (!route_only && h->test_timeout_pending) ? 1 : 0;
    if (a.test_timeout) h->test_timeout_pending = false;
    a.wait_ns = 1000000000ll;
    a.trace = h->trace;
    a.trace_units = h->trace_units;
    return a;
}

// One cooperative launch (all CTAs resident: one per SM) of the batched-GEMV kernel.
ds4moe_status launch_decode(ds4moe *h, const void *x, int T, float *y, cudaStream_t st, bool route_only) {
    const DecArgs a = decode_args(h, x, T, y, route_only);
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(h->num_sms);
    lc.blockDim = dim3(DK_THREADS);
    lc.dynamicSmemBytes = DK_SMEM;
    lc.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    // the one-token build only for one token (its consumers assume one token per group)
    if (h->trace) CK(h, cudaLaunchKernelEx(&lc, decode_kernel<true, false>, a));
    else if (T == 1) CK(h, cudaLaunchKernelEx(&lc, decode_kernel<false, true>, a));
    else CK(h, cudaLaunchKernelEx(&lc, decode_kernel<false, false>, a));
    return DS4MOE_OK;
}

template <int NPL>
void launch_topk_block(ds4moe *h, const void *x, int T, cudaStream_t st) {
    const ds4moe_config &g = h->cfg;
    topk_block_kernel<NPL><<<(T + 63) / 64, TOPK_THREADS, 0, st>>>(
        h->logits, h->labs, T, g.n_experts, g.top_k, g.hidden, BOUND_MMA, reinterpret_cast<const __nv_bfloat16 *>(x),
        h->wr, h->has_bias ? h->bias : nullptr, h->ro, h->blk_cnt, h->blk_mask);
}

void record(ds4moe *h, cudaStream_t st) {
    if ((h->cfg.flags & DS4MOE_FLAG_PROFILE) && h->n_ev < 9) cudaEventRecord(h->ev[h->n_ev++], st);
}

bool use_decode(const ds4moe *h, int T) {
    if (T > MAX_DECODE_T) return false;
    if (h->cfg.flags & DS4MOE_FLAG_FORCE_PREFILL) return false;
    return true;
}

// Routing of T tokens into the workspace (top-k, weights, permutation, active list).
ds4moe_status route_impl(ds4moe *h, const void *x, int T, cudaStream_t st, bool decode) {
    const ds4moe_config &g = h->cfg;
    if (decode) {
        ds4moe_status r = launch_decode(h, x, T, nullptr, st, true);
        record(h, st);
        return r;
    }
    if (!h->maps_ok) return fail(h, DS4MOE_ECUDA, "tensor maps unavailable (cuTensorMapEncodeTiled)");
    CUtensorMap tm_xr{};
    if (!make_map(&tm_xr, x, g.hidden, (uint64_t)T, RM_N, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16))
        return fail(h, DS4MOE_ECUDA, "tensor map of x");
    RouterArgs ra{};
    ra.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    ra.T = T; ra.H = g.hidden; ra.E = g.n_experts;
    ra.bias = h->has_bias ? h->bias : nullptr;
    ra.wr_norm = h->wr_norm;
    ra.logits = h->logits; ra.labs = h->labs;
    ra.status = h->status; ra.dbg = h->dbg;
    const dim3 grid((T + RM_N - 1) / RM_N, (g.n_experts + RM_M - 1) / RM_M);
    router_mma_kernel<<<grid, RM_THREADS, RM_SMEM, st>>>(h->tm_wr, tm_xr, ra);
    CKL(h);
    switch (npl_of(g.n_experts)) {
        case 1: launch_topk_block<1>(h, x, T, st); break;
        case 2: launch_topk_block<2>(h, x, T, st); break;
        case 4: launch_topk_block<4>(h, x, T, st); break;
        default: launch_topk_block<8>(h, x, T, st); break;
    }
    CKL(h);
    permute_scatter_kernel<<<(T + 63) / 64, 256, 0, st>>>(h->blk_cnt, h->blk_mask, (T + 63) / 64, T, g.n_experts,
                                                          g.top_k, h->ro);
    CKL(h);
    record(h, st);
    return DS4MOE_OK;
}

// Batched-GEMV path: one launch does the routing and the whole layer.
ds4moe_status forward_decode(ds4moe *h, const void *x, int T, float *y, cudaStream_t st) {
    ds4moe_status r = launch_decode(h, x, T, y, st, false);
    record(h, st);
    return r;
}

// Grouped tensor-core path: prefill routing, gather of the activations in pair order (plus
// the tokens for the shared expert), tile lists, GEMM1 (gate/up + SwiGLU), GEMM2 (down,
// scaled by the routing weights), combine.
ds4moe_status forward_prefill(ds4moe *h, const void *x, int T, float *y, cudaStream_t st) {
    const ds4moe_config &g = h->cfg;
    if (!h->maps_ok) return fail(h, DS4MOE_ECUDA, "tensor maps unavailable (cuTensorMapEncodeTiled)");
    ds4moe_status r = route_impl(h, x, T, st, false);
    if (r != DS4MOE_OK) return r;
    const int P = T * g.top_k, Is = g.shared_inter;
    PrefillWork &w = h->pw;
    pf_gather_kernel<<<P + (Is > 0 ? T : 0), 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), T, g.hidden,
                                                          g.top_k, h->ro.sorted_token, h->ro.sorted_slot,
                                                          h->ro.topk_w, P, w.xall, w.row_w, h->status);
    CKL(h);
    pf_build_tiles_kernel<<<1, 256, 0, st>>>(h->ro.offsets, h->ro.active, h->ro.n_active, T, P, PF_N1, g.inter,
                                             g.hidden, Is, g.hidden, w.tiles1, w.n_tiles, w.max_tiles1);
    CKL(h);
    pf_build_tiles_kernel<<<1, 256, 0, st>>>(h->ro.offsets, h->ro.active, h->ro.n_active, T, P, PF_N2, g.hidden,
                                             g.inter, Is > 0 ? g.hidden : 0, Is, w.tiles2, w.n_tiles + 1, w.max_tiles2);
    CKL(h);
    record(h, st);
    PfArgs a1{};
    a1.tiles = w.tiles1; a1.n_tiles = w.n_tiles; a1.gemm = 1;
    a1.wq0 = h->gate; a1.wq1 = h->up; a1.wq_bytes = h->gu_bytes;
    const size_t rows = (size_t)g.max_tokens * g.top_k + g.max_tokens;
    a1.out16 = w.hall; a1.ld_out = w.ldH; a1.status = h->status;
    a1.out_elems = rows * w.ldH; a1.wq_total = (size_t)g.n_experts * h->gu_bytes; a1.b_rows_total = (int)rows;
    a1.dbg = h->dbg;
    pf_gemm_kernel<1><<<h->num_sms, PF_THREADS, PfCfg<1>::SMEM, st>>>(h->tm_x, Is > 0 ? h->tm_sg : h->tm_x,
                                                           Is > 0 ? h->tm_su : h->tm_x, a1);
    CKL(h);
    record(h, st);
    PfArgs a2{};
    a2.tiles = w.tiles2; a2.n_tiles = w.n_tiles + 1; a2.gemm = 2;
    a2.wq0 = h->down; a2.wq1 = nullptr; a2.wq_bytes = h->d_bytes;
    a2.out32 = w.oall; a2.ld_out = g.hidden; a2.row_scale = w.row_w; a2.status = h->status;
    a2.out_elems = rows * g.hidden; a2.wq_total = (size_t)g.n_experts * h->d_bytes; a2.b_rows_total = (int)rows;
    a2.dbg = h->dbg;
    pf_gemm_kernel<2><<<h->num_sms, PF_THREADS, PfCfg<2>::SMEM, st>>>(h->tm_h, Is > 0 ? h->tm_sd : h->tm_h,
                                                           Is > 0 ? h->tm_sd : h->tm_h, a2);
    CKL(h);
    record(h, st);
    pf_combine_kernel<<<T, 256, 0, st>>>(w.oall, T, g.hidden, g.top_k, h->ro.inv_pos, P, Is > 0 ? 1 : 0, y);
    CKL(h);
    record(h, st);
    return DS4MOE_OK;
}

ds4moe_status check_x(ds4moe *h, const void *x, int T) {
    if (!h) return DS4MOE_EINVAL;
    if (injected("launch")) return fail(h, DS4MOE_ECUDA, "kernel launch failed (injected: DS4MOE_FAULT=launch)");
    if (!h->loaded) return fail(h, DS4MOE_ESTATE, "no weights loaded");
    if (T < 0 || T > h->cfg.max_tokens) return fail(h, DS4MOE_EINVAL, "T=%d outside [0, max_tokens=%d]", T, h->cfg.max_tokens);
    if (T > 0 && (!x || !aligned16(x))) return fail(h, DS4MOE_EINVAL, "x must be a 16-byte aligned device pointer");
    return DS4MOE_OK;
}

// ------------------------------------------------------- routing with static scratch
// Scratch of ds4moe_route_static, one array per device (a file-scope __device__ array lives
// in every device's copy of this module).  Carved as: fp64 logits [T][E], fp32 error
// bounds [T][E], per-64-token block counts [NB][E] and masks [NB][E], the active-expert
// list [E] and its length, for T <= DS4MOE_ROUTE_STATIC_MAX_TOKENS and E <= 256.  Every
// word is written before it is read within one call, so nothing has to start at zero.
constexpr int RS_MAX_T = DS4MOE_ROUTE_STATIC_MAX_TOKENS;
constexpr int RS_MAX_NB = (RS_MAX_T + 63) / 64;
constexpr size_t RS_LOGITS = (size_t)RS_MAX_T * MAX_EXPERTS * sizeof(double);
constexpr size_t RS_LABS = (size_t)RS_MAX_T * MAX_EXPERTS * sizeof(float);
constexpr size_t RS_CNT = (size_t)RS_MAX_NB * MAX_EXPERTS * sizeof(int);
constexpr size_t RS_MASK = (size_t)RS_MAX_NB * MAX_EXPERTS * sizeof(unsigned long long);
constexpr size_t RS_ACTIVE = (size_t)MAX_EXPERTS * sizeof(int);
constexpr size_t RS_BYTES = RS_LOGITS + RS_LABS + RS_CNT + RS_MASK + RS_ACTIVE + 256;
static_assert(RS_LOGITS % 256 == 0 && RS_LABS % 256 == 0 && RS_CNT % 256 == 0 && RS_MASK % 256 == 0 &&
                  RS_ACTIVE % 256 == 0,
              "scratch pieces keep 256-byte alignment");
static __device__ __align__(256) unsigned char g_route_scratch[RS_BYTES];

constexpr int RS_MAX_DEVICES = 64;
std::mutex g_rs_mutex;
void *g_rs_addr[RS_MAX_DEVICES] = {};

// Device address of the scratch on h's device, resolved once per device with that device
// current (the caller has made it current).
ds4moe_status route_static_scratch(ds4moe *h, unsigned char **out) {
    if (h->device < 0 || h->device >= RS_MAX_DEVICES)
        return fail(h, DS4MOE_EINVAL, "device %d is beyond the static scratch table", h->device);
    std::lock_guard<std::mutex> lock(g_rs_mutex);
    if (!g_rs_addr[h->device]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || !p)
            return fail(h, DS4MOE_ECUDA, "cudaGetSymbolAddress of the routing scratch: %s", cudaGetErrorString(e));
        g_rs_addr[h->device] = p;
    }
    *out = static_cast<unsigned char *>(g_rs_addr[h->device]);
    return DS4MOE_OK;
}

}  // namespace

extern "C" {

const char *ds4moe_status_string(ds4moe_status s) {
    switch (s) {
        case DS4MOE_OK: return "ok";
        case DS4MOE_EINVAL: return "invalid argument";
        case DS4MOE_ENOMEM: return "out of memory";
        case DS4MOE_ECUDA: return "CUDA error";
        case DS4MOE_ESTATE: return "invalid state";
        case DS4MOE_ETIMEOUT: return "device-side wait timed out";
        case DS4MOE_EDEVICE: return "device-side check failed";
    }
    return "unknown status";
}

const char *ds4moe_last_error(const ds4moe *h) { return h ? h->err.c_str() : "null handle"; }

ds4moe_status ds4moe_create(const ds4moe_config *cfg, int cuda_device, ds4moe **out) {
    if (!cfg || !out) return DS4MOE_EINVAL;
    *out = nullptr;
    const ds4moe_config &g = *cfg;
    if (g.hidden < 256 || g.hidden > 16384 || g.hidden % 256) return DS4MOE_EINVAL;
    if (g.inter < 256 || g.inter > 16384 || g.inter % 256) return DS4MOE_EINVAL;
    if (g.shared_inter < 0 || g.shared_inter > 16384 || g.shared_inter % 256) return DS4MOE_EINVAL;
    if (g.n_experts < 1 || g.n_experts > MAX_EXPERTS) return DS4MOE_EINVAL;
    if (g.top_k < 1 || g.top_k > MAX_TOPK || g.top_k > g.n_experts) return DS4MOE_EINVAL;
    if (g.max_tokens < 1 || g.max_tokens > 65536) return DS4MOE_EINVAL;
    if (injected("alloc")) return DS4MOE_ENOMEM;
    ds4moe *h = new ds4moe();
    h->cfg = g;
    h->device = cuda_device;
    h->test_timeout_pending = (g.flags & DS4MOE_FLAG_TEST_TIMEOUT) != 0;
    cudaError_t e = cudaSetDevice(cuda_device);
    if (e != cudaSuccess) {
        delete h;
        return DS4MOE_ECUDA;
    }
    cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, cuda_device);
    Carver sizer{nullptr};
    layout_workspace(h, sizer);
    h->ws_bytes = sizer.off + 256;
    e = cudaMalloc(&h->ws, h->ws_bytes);
    if (e != cudaSuccess) {
        delete h;
        return e == cudaErrorMemoryAllocation ? DS4MOE_ENOMEM : DS4MOE_ECUDA;
    }
    Carver c{reinterpret_cast<char *>(h->ws)};
    layout_workspace(h, c);
    h->ro.fallbacks = h->fallbacks;
    h->ro.status = h->status;
    cudaMemset(h->ws, 0, h->ws_bytes);
    if (g.flags & DS4MOE_FLAG_TRACE) {
        h->trace_units = decode_unit_bound(g, std::min(g.max_tokens, MAX_DECODE_T));
        const size_t words = 12 * (size_t)h->trace_units + 8 * (size_t)h->num_sms + 16;
        if (cudaMalloc(&h->trace, words * 8) != cudaSuccess) {
            cudaFree(h->ws);
            delete h;
            return DS4MOE_ENOMEM;
        }
        cudaMemset(h->trace, 0, words * 8);
    }
    cudaFuncSetAttribute(decode_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DK_SMEM);
    cudaFuncSetAttribute(decode_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DK_SMEM);
    cudaFuncSetAttribute(decode_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DK_SMEM);
    {   // the batched-GEMV kernel is a cooperative launch of one CTA per SM (every build)
        int per_sm = 0, m = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<false, false>, DK_THREADS, DK_SMEM);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, decode_kernel<false, true>, DK_THREADS, DK_SMEM);
        per_sm = std::min(per_sm, m);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, decode_kernel<true, false>, DK_THREADS, DK_SMEM);
        per_sm = std::min(per_sm, m);
        if (per_sm < 1) {
            cudaGetLastError();
            ds4moe_destroy(h);
            return DS4MOE_ECUDA;
        }
    }
    prefill_init(h->pw);
    cudaFuncSetAttribute(pf_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PfCfg<1>::SMEM);
    cudaFuncSetAttribute(pf_gemm_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PfCfg<2>::SMEM);
    cudaFuncSetAttribute(router_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RM_SMEM);
    for (auto &ev : h->ev) cudaEventCreate(&ev);
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        ds4moe_destroy(h);
        return DS4MOE_ECUDA;
    }
    *out = h;
    return DS4MOE_OK;
}

void ds4moe_destroy(ds4moe *h) {
    if (!h) return;
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    free_weights(h);
    if (h->ws) cudaFree(h->ws);
    if (h->trace) cudaFree(h->trace);
    for (auto &ev : h->ev)
        if (ev) cudaEventDestroy(ev);
    delete h;
}

ds4moe_status ds4moe_load_q2k_experts(ds4moe *h, const void *gate_q2k, const void *up_q2k, const void *down_q2k,
                                      const uint16_t *router_w_bf16, const float *router_bias,
                                      const uint16_t *shared_gate_bf16, const uint16_t *shared_up_bf16,
                                      const uint16_t *shared_down_bf16, void *cuda_stream) {
    if (!h) return DS4MOE_EINVAL;
    const ds4moe_config &g = h->cfg;
    if (!gate_q2k || !up_q2k || !down_q2k || !router_w_bf16) return fail(h, DS4MOE_EINVAL, "null weight pointer");
    if (g.shared_inter > 0 && (!shared_gate_bf16 || !shared_up_bf16 || !shared_down_bf16))
        return fail(h, DS4MOE_EINVAL, "shared expert weights missing");
    if (injected("h2d")) return fail(h, DS4MOE_ECUDA, "host-to-device copy failed (injected: DS4MOE_FAULT=h2d)");
    CK(h, cudaSetDevice(h->device));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    free_weights(h);
    const size_t E = g.n_experts, H = g.hidden, I = g.inter, Is = g.shared_inter;
    h->gu_bytes = tiled_bytes((int)I, (int)H);
    h->d_bytes = tiled_bytes((int)H, (int)I);
    CK(h, cudaMalloc(&h->gate, E * h->gu_bytes));
    CK(h, cudaMalloc(&h->up, E * h->gu_bytes));
    CK(h, cudaMalloc(&h->down, E * h->d_bytes));
    CK(h, cudaMalloc(&h->wr, E * H * 2));
    CK(h, cudaMalloc(&h->bias, E * 4));
    CK(h, cudaMalloc(&h->wr_norm, E * 4));
    if (Is) {
        CK(h, cudaMalloc(&h->sg, Is * H * 2));
        CK(h, cudaMalloc(&h->su, Is * H * 2));
        CK(h, cudaMalloc(&h->sd, H * Is * 2));
    }
    // stage the AoS blocks through a bounded device buffer, one group of experts at a time
    const size_t stage_cap = (size_t)256 << 20;
    uint8_t *stage = nullptr;
    CK(h, cudaMalloc(&stage, std::min(stage_cap, std::max(h->gu_bytes, h->d_bytes))));
    struct M { const void *src; uint8_t *dst; size_t bytes; int rows, nb; };
    const M mats[3] = {{gate_q2k, h->gate, h->gu_bytes, (int)I, (int)(H / QK)},
                       {up_q2k, h->up, h->gu_bytes, (int)I, (int)(H / QK)},
                       {down_q2k, h->down, h->d_bytes, (int)H, (int)(I / QK)}};
    for (const M &m : mats) {
        const size_t per = std::max<size_t>(1, std::min(stage_cap, std::max(h->gu_bytes, h->d_bytes)) / m.bytes);
        for (size_t e0 = 0; e0 < E; e0 += per) {
            const size_t ne = std::min(per, E - e0);
            cudaError_t ce = cudaMemcpyAsync(stage, (const uint8_t *)m.src + e0 * m.bytes, ne * m.bytes,
                                             cudaMemcpyHostToDevice, st);
            if (ce != cudaSuccess) { cudaFree(stage); return fail(h, DS4MOE_ECUDA, "weight upload: %s", cudaGetErrorString(ce)); }
            const long long n = (long long)ne * m.rows * m.nb;
            const int grid = (int)std::min<long long>((n + 255) / 256, 65536);
            repack_q2k_kernel<<<grid, 256, 0, st>>>(stage, m.dst + e0 * m.bytes, (int)ne, m.rows, m.nb);
            ce = cudaGetLastError();
            if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
            if (ce != cudaSuccess) { cudaFree(stage); return fail(h, DS4MOE_ECUDA, "repack: %s", cudaGetErrorString(ce)); }
        }
    }
    cudaFree(stage);
    CK(h, cudaMemcpy(h->wr, router_w_bf16, E * H * 2, cudaMemcpyHostToDevice));
    std::vector<float> norms(E), b(E, 0.0f);
    for (size_t e = 0; e < E; ++e) {
        double ss = 0.0;
        for (size_t i = 0; i < H; ++i) {
            uint32_t u = (uint32_t)router_w_bf16[e * H + i] << 16;
            float f;
            memcpy(&f, &u, 4);
            ss += (double)f * (double)f;
        }
        norms[e] = nextafterf((float)std::sqrt(ss), INFINITY);
        if (router_bias) b[e] = router_bias[e];
    }
    h->has_bias = router_bias != nullptr;
    CK(h, cudaMemcpy(h->wr_norm, norms.data(), E * 4, cudaMemcpyHostToDevice));
    CK(h, cudaMemcpy(h->bias, b.data(), E * 4, cudaMemcpyHostToDevice));
    if (Is) {
        CK(h, cudaMemcpy(h->sg, shared_gate_bf16, Is * H * 2, cudaMemcpyHostToDevice));
        CK(h, cudaMemcpy(h->su, shared_up_bf16, Is * H * 2, cudaMemcpyHostToDevice));
        CK(h, cudaMemcpy(h->sd, shared_down_bf16, H * Is * 2, cudaMemcpyHostToDevice));
    }
    if (Is) {
        CK(h, cudaMalloc(&h->sg16, Is * H * 2));
        CK(h, cudaMalloc(&h->su16, Is * H * 2));
        CK(h, cudaMalloc(&h->sd16, H * Is * 2));
        bf16_to_f16_kernel<<<1024, 256>>>(h->sg, h->sg16, Is * H);
        bf16_to_f16_kernel<<<1024, 256>>>(h->su, h->su16, Is * H);
        bf16_to_f16_kernel<<<1024, 256>>>(h->sd, h->sd16, H * Is);
        CK(h, cudaGetLastError());
    }
    CK(h, cudaDeviceSynchronize());
    {
        const uint64_t rows = (uint64_t)g.max_tokens * g.top_k + g.max_tokens;
        bool ok = make_map(&h->tm_x, h->pw.xall, H, rows, PF_BBOX) && make_map(&h->tm_h, h->pw.hall, h->pw.ldH, rows, PF_BBOX) &&
                  make_map(&h->tm_wr, h->wr, H, E, RM_M, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
        if (Is) {
            ok = ok && make_map(&h->tm_sg, h->sg16, H, Is, PF_M) && make_map(&h->tm_su, h->su16, H, Is, PF_M) &&
                 make_map(&h->tm_sd, h->sd16, Is, H, PF_M);
        }
        h->maps_ok = ok;
    }
    h->loaded = true;
    h->last_stream = st;
    return DS4MOE_OK;
}

ds4moe_status ds4moe_route(ds4moe *h, const void *x_bf16_dev, int32_t T, int32_t *topk_idx_dev, float *topk_w_dev,
                           int32_t *expert_offsets_dev, int32_t *sorted_token_dev, int32_t *sorted_slot_dev,
                           int32_t *inv_pos_dev, void *cuda_stream) {
    ds4moe_status r = check_x(h, x_bf16_dev, T);
    if (r != DS4MOE_OK) return r;
    if (T == 0) return DS4MOE_OK;
    if (!topk_idx_dev || !topk_w_dev) return fail(h, DS4MOE_EINVAL, "topk outputs are required");
    CK(h, cudaSetDevice(h->device));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    h->last_stream = st;
    h->n_ev = 0;
    r = route_impl(h, x_bf16_dev, T, st, use_decode(h, T));
    if (r != DS4MOE_OK) return r;
    const ds4moe_config &g = h->cfg;
    const size_t P = (size_t)T * g.top_k;
    CK(h, cudaMemcpyAsync(topk_idx_dev, h->ro.topk_idx, P * 4, cudaMemcpyDeviceToDevice, st));
    CK(h, cudaMemcpyAsync(topk_w_dev, h->ro.topk_w, P * 4, cudaMemcpyDeviceToDevice, st));
    if (expert_offsets_dev)
        CK(h, cudaMemcpyAsync(expert_offsets_dev, h->ro.offsets, (g.n_experts + 1) * 4, cudaMemcpyDeviceToDevice, st));
    if (sorted_token_dev) CK(h, cudaMemcpyAsync(sorted_token_dev, h->ro.sorted_token, P * 4, cudaMemcpyDeviceToDevice, st));
    if (sorted_slot_dev) CK(h, cudaMemcpyAsync(sorted_slot_dev, h->ro.sorted_slot, P * 4, cudaMemcpyDeviceToDevice, st));
    if (inv_pos_dev) CK(h, cudaMemcpyAsync(inv_pos_dev, h->ro.inv_pos, P * 4, cudaMemcpyDeviceToDevice, st));
    return DS4MOE_OK;
}

ds4moe_status ds4moe_forward(ds4moe *h, const void *x_bf16_dev, int32_t T, float *y_f32_dev, void *cuda_stream) {
    ds4moe_status r = check_x(h, x_bf16_dev, T);
    if (r != DS4MOE_OK) return r;
    if (T == 0) return DS4MOE_OK;
    if (!y_f32_dev || !aligned16(y_f32_dev)) return fail(h, DS4MOE_EINVAL, "y must be a 16-byte aligned device pointer");
    CK(h, cudaSetDevice(h->device));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    h->last_stream = st;
    h->n_ev = 0;
    record(h, st);
    const bool dec = use_decode(h, T);
    h->last_path = dec ? 1 : 2;
    h->last_T = T;
    if (dec) return forward_decode(h, x_bf16_dev, T, y_f32_dev, st);
    return forward_prefill(h, x_bf16_dev, T, y_f32_dev, st);
}

ds4moe_status ds4moe_forward_host(ds4moe *h, const uint16_t *x_bf16, int32_t T, float *y_f32, void *cuda_stream) {
    if (!h) return DS4MOE_EINVAL;
    if (T < 0 || T > h->cfg.max_tokens) return fail(h, DS4MOE_EINVAL, "T out of range");
    if (T == 0) return DS4MOE_OK;
    if (!x_bf16 || !y_f32) return fail(h, DS4MOE_EINVAL, "null host buffer");
    CK(h, cudaSetDevice(h->device));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    const size_t H = h->cfg.hidden;
    // On the batched-GEMV path a page-locked, device-mapped y is written by the kernel
    // itself (its last writes cross to the host; no separate copy).  Other buffers go
    // through the handle's staging buffer and one copy back.
    float *y_direct = nullptr;
    if (use_decode(h, T)) {
        cudaPointerAttributes pa{};
        if (cudaPointerGetAttributes(&pa, y_f32) == cudaSuccess && pa.type == cudaMemoryTypeHost &&
            pa.devicePointer && aligned16(pa.devicePointer))
            y_direct = static_cast<float *>(pa.devicePointer);
        cudaGetLastError();   // an unregistered pointer is not an error here
    }
    CK(h, cudaMemcpyAsync(h->x_stage, x_bf16, (size_t)T * H * 2, cudaMemcpyHostToDevice, st));
    ds4moe_status r = ds4moe_forward(h, h->x_stage, T, y_direct ? y_direct : h->y_stage, cuda_stream);
    if (r != DS4MOE_OK) return r;
    if (!y_direct) CK(h, cudaMemcpyAsync(y_f32, h->y_stage, (size_t)T * H * 4, cudaMemcpyDeviceToHost, st));
    CK(h, cudaStreamSynchronize(st));
    return DS4MOE_OK;
}

ds4moe_status ds4moe_rms_renorm(const float *y_f32_dev, int32_t T, int32_t H, uint16_t *x_bf16_dev, void *cuda_stream) {
    if (T < 0 || H <= 0 || (T > 0 && (!y_f32_dev || !x_bf16_dev))) return DS4MOE_EINVAL;
    if (T == 0) return DS4MOE_OK;
    rms_renorm_kernel<<<T, 256, 0, reinterpret_cast<cudaStream_t>(cuda_stream)>>>(
        y_f32_dev, H, reinterpret_cast<__nv_bfloat16 *>(x_bf16_dev));
    return cudaGetLastError() == cudaSuccess ? DS4MOE_OK : DS4MOE_ECUDA;
}

ds4moe_status ds4moe_score_eval(const float *logits_dev, int32_t n, float *scores_dev, int32_t variant, void *cuda_stream) {
    if (n < 0 || (n > 0 && (!logits_dev || !scores_dev)) || variant < 0 || variant > 1) return DS4MOE_EINVAL;
    if (n == 0) return DS4MOE_OK;
    score_eval_kernel<<<(n + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(cuda_stream)>>>(logits_dev, n, scores_dev,
                                                                                                 variant);
    return cudaGetLastError() == cudaSuccess ? DS4MOE_OK : DS4MOE_ECUDA;
}

ds4moe_status ds4moe_export_q2k(ds4moe *h, int32_t which, int32_t expert, void *out) {
    if (!h) return DS4MOE_EINVAL;
    if (!h->loaded) return fail(h, DS4MOE_ESTATE, "no weights loaded");
    if (which < 0 || which > 2 || expert < 0 || expert >= h->cfg.n_experts || !out)
        return fail(h, DS4MOE_EINVAL, "bad export arguments");
    CK(h, cudaSetDevice(h->device));
    const int rows = which == 2 ? h->cfg.hidden : h->cfg.inter;
    const int K = which == 2 ? h->cfg.inter : h->cfg.hidden;
    const size_t bytes = which == 2 ? h->d_bytes : h->gu_bytes;
    const uint8_t *src = (which == 0 ? h->gate : which == 1 ? h->up : h->down) + (size_t)expert * bytes;
    uint8_t *tmp = nullptr;
    CK(h, cudaMalloc(&tmp, bytes));
    const long long n = (long long)rows * (K / QK);
    export_q2k_kernel<<<(int)std::min<long long>((n + 255) / 256, 65536), 256>>>(src, tmp, rows, K / QK);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaMemcpy(out, tmp, bytes, cudaMemcpyDeviceToHost);
    cudaFree(tmp);
    if (e != cudaSuccess) return fail(h, DS4MOE_ECUDA, "export: %s", cudaGetErrorString(e));
    return DS4MOE_OK;
}

ds4moe_status ds4moe_sync_status(ds4moe *h) {
    if (!h) return DS4MOE_EINVAL;
    CK(h, cudaSetDevice(h->device));
    CK(h, cudaStreamSynchronize(h->last_stream));
    int st = 0;
    CK(h, cudaMemcpy(&st, h->status, 4, cudaMemcpyDeviceToHost));
    if (st != 0) {
        const int zero = 0;
        int dbg[8] = {};
        cudaMemcpy(dbg, h->dbg, sizeof dbg, cudaMemcpyDeviceToHost);
        cudaMemset(h->dbg, 0, sizeof dbg);
        CK(h, cudaMemcpy(h->status, &zero, 4, cudaMemcpyHostToDevice));
        CK(h, cudaMemset(h->ctl, 0, sizeof(DecCtl)));
        return fail(h, (ds4moe_status)st, "device status %d (check %d: tile %d, %d %d %d %d, cta %d, thread %d)", st,
                    dbg[0], dbg[1], dbg[2], dbg[3], dbg[4], dbg[5], dbg[6], dbg[7]);
    }
    return DS4MOE_OK;
}

ds4moe_status ds4moe_get_trace(ds4moe *h, int64_t *out, int32_t max_records, int32_t *n_records,
                               int32_t *unit_bounds) {
    if (!h || !n_records) return DS4MOE_EINVAL;
    if (!h->trace) return fail(h, DS4MOE_ESTATE, "handle was created without DS4MOE_FLAG_TRACE");
    ds4moe_status r = ds4moe_sync_status(h);
    const size_t words = 12 * (size_t)h->trace_units + 8 * (size_t)h->num_sms + 16;
    std::vector<unsigned long long> buf(words);
    CK(h, cudaMemcpy(buf.data(), h->trace, words * 8, cudaMemcpyDeviceToHost));
    const int n = std::min<int>(max_records, (int)(words / 4));
    if (out && n > 0) memcpy(out, buf.data(), (size_t)n * 32);
    *n_records = n;
    if (unit_bounds) {
        // the first unit of each of the four phases and the end of the last launch (written
        // by the routing step of CTA 0), then the numbers of unit and CTA records
        const unsigned long long *b = buf.data() + 4 * (size_t)h->trace_units + 8 * (size_t)h->num_sms;
        unit_bounds[0] = 0;
        for (int i = 0; i < 4; ++i) unit_bounds[1 + i] = (int32_t)b[i];
        unit_bounds[5] = h->trace_units;
        unit_bounds[6] = h->num_sms;
    }
    return r;
}

ds4moe_status ds4moe_get_stats(ds4moe *h, ds4moe_stats *out) {
    if (!h || !out) return DS4MOE_EINVAL;
    ds4moe_status r = ds4moe_sync_status(h);
    memset(out, 0, sizeof *out);
    unsigned long long fb = 0;
    CK(h, cudaMemcpy(&fb, h->fallbacks, 8, cudaMemcpyDeviceToHost));
    out->router_fallback_tokens = (int64_t)fb;
    out->last_path = h->last_path;
    out->last_tokens = h->last_T;
    if ((h->cfg.flags & DS4MOE_FLAG_PROFILE) && h->n_ev > 1) {
        out->n_stages = std::min(h->n_ev - 1, 8);
        for (int i = 0; i < out->n_stages; ++i) cudaEventElapsedTime(&out->stage_ms[i], h->ev[i], h->ev[i + 1]);
    }
    return r;
}

ds4moe_status ds4moe_route_static(ds4moe *h, const void *x_bf16_dev, int32_t T, int32_t *topk_idx_dev,
                                  float *topk_w_dev, int32_t *expert_offsets_dev, int32_t *sorted_token_dev,
                                  int32_t *sorted_slot_dev, int32_t *inv_pos_dev, void *cuda_stream) {
    ds4moe_status r = check_x(h, x_bf16_dev, T);
    if (r != DS4MOE_OK) return r;
    if (T > RS_MAX_T)
        return fail(h, DS4MOE_EINVAL, "T=%d exceeds the %d tokens of the static routing scratch", T, RS_MAX_T);
    if (T == 0) return DS4MOE_OK;
    if (!topk_idx_dev || !topk_w_dev || !expert_offsets_dev || !sorted_token_dev || !sorted_slot_dev || !inv_pos_dev)
        return fail(h, DS4MOE_EINVAL, "every output of ds4moe_route_static is required");
    CK(h, cudaSetDevice(h->device));
    unsigned char *scratch = nullptr;
    r = route_static_scratch(h, &scratch);
    if (r != DS4MOE_OK) return r;
    const ds4moe_config &g = h->cfg;
    const int E = g.n_experts, NB = (T + 63) / 64;
    double *logits = reinterpret_cast<double *>(scratch);
    float *labs = reinterpret_cast<float *>(scratch + RS_LOGITS);
    int *blk_cnt = reinterpret_cast<int *>(scratch + RS_LOGITS + RS_LABS);
    unsigned long long *blk_mask = reinterpret_cast<unsigned long long *>(scratch + RS_LOGITS + RS_LABS + RS_CNT);
    int *active = reinterpret_cast<int *>(scratch + RS_LOGITS + RS_LABS + RS_CNT + RS_MASK);
    RouteOut ro = h->ro;   // the handle's fallback counter and status word; outputs are the caller's
    ro.topk_idx = topk_idx_dev;
    ro.topk_w = topk_w_dev;
    ro.offsets = expert_offsets_dev;
    ro.sorted_token = sorted_token_dev;
    ro.sorted_slot = sorted_slot_dev;
    ro.inv_pos = inv_pos_dev;
    ro.active = active;
    ro.n_active = active + MAX_EXPERTS;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(cuda_stream);
    h->last_stream = st;
    h->n_ev = 0;
    const __nv_bfloat16 *xb = reinterpret_cast<const __nv_bfloat16 *>(x_bf16_dev);
    dim3 grid((T + PR_T - 1) / PR_T, (E + PR_E - 1) / PR_E);
    router_gemm_kernel<<<grid, 128, 0, st>>>(xb, T, g.hidden, h->wr, E, h->has_bias ? h->bias : nullptr, h->wr_norm,
                                             logits, labs);
    CKL(h);
    const float *bias = h->has_bias ? h->bias : nullptr;
    switch (npl_of(E)) {
        case 1: topk_block_kernel<1><<<NB, TOPK_THREADS, 0, st>>>(logits, labs, T, E, g.top_k, g.hidden, BOUND_CHUNK32, xb, h->wr, bias, ro, blk_cnt, blk_mask); break;
        case 2: topk_block_kernel<2><<<NB, TOPK_THREADS, 0, st>>>(logits, labs, T, E, g.top_k, g.hidden, BOUND_CHUNK32, xb, h->wr, bias, ro, blk_cnt, blk_mask); break;
        case 4: topk_block_kernel<4><<<NB, TOPK_THREADS, 0, st>>>(logits, labs, T, E, g.top_k, g.hidden, BOUND_CHUNK32, xb, h->wr, bias, ro, blk_cnt, blk_mask); break;
        default: topk_block_kernel<8><<<NB, TOPK_THREADS, 0, st>>>(logits, labs, T, E, g.top_k, g.hidden, BOUND_CHUNK32, xb, h->wr, bias, ro, blk_cnt, blk_mask); break;
    }
    CKL(h);
    permute_scatter_kernel<<<NB, 256, 0, st>>>(blk_cnt, blk_mask, NB, T, E, g.top_k, ro);
    CKL(h);
    return DS4MOE_OK;
}

}  // extern "C"
