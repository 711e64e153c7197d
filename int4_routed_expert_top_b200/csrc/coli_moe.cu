// coli_moe.cu - C ABI of libcolimoe (see include/coli_moe.h).
//
// Host code validates arguments, plans the caller's workspace and launches the
// kernels of route.cuh, gemv.cuh, gemm.cuh and misc.cuh on the caller's
// stream.  Nothing here synchronises the host or allocates device memory.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>
#include <string>

#include "coli_moe.h"
#include "common.cuh"
#include "fused.cuh"
#include "gemm.cuh"
#include "gemv.cuh"
#include "misc.cuh"
#include "route.cuh"
#include "split.cuh"

using namespace coli;

struct coli_moe_layer {
    coli_moe_desc d;       // as created
    int bits;              // 4 or 8 (bits per weight code)
    BlobLayout L;
    // what a forward computes: d with n_shared = 0 on a handle restricted to a
    // range of routed experts without the shared ones; where the blobs sit;
    // which picks are computed (top-p, expert range)
    coli_moe_desc run;
    ExpertStore store;
    PickFilter filter;
    // test of the bounded waits (coli_moe_layer_set_wait_test)
    int withhold = -1;
};

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int check_launch(const char* what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(COLI_E_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return COLI_OK;
}

cudaStream_t S(coli_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

bool shape_ok(int H, int I, int group) {
    return H > 0 && I > 0 && H % 128 == 0 && I % 128 == 0 && (group == 0 || group == 64);
}

// ---------------------------------------------------------------------------
// workspace plan
// ---------------------------------------------------------------------------
struct WsPlan {
    int64_t zpart, idx, w, offsets, pair_tok, pair_slot, uniq, n_uniq, inv;
    int64_t unit_expert, unit_begin, unit_end, n_units, counters, err;
    int64_t xq, xinv, hq, hinv, o, xg, hg, hmax, hsc;
    int64_t xq8, part, queue, sel;  // fused small-batch kernel (T <= kFzMaxT only)
    int64_t hrec, squeue;           // two-pass path (xq8 as well)
    int64_t total;
};

// workspace layouts: the GEMV/GEMM base, the base with the fused path's
// buffers where that path applies (else with the two-pass path's), the base
// with the two-pass path's buffers.  Where the fused path applies its buffers
// are larger than the two-pass path's, so the full layout covers every path.
enum PlanKind { kPlanBase = 0, kPlanFull = 1, kPlanSplit = 2 };

bool fused_fits(const coli_moe_desc& d, int T) {
    return T <= kFzMaxT && T * (d.k + d.n_shared) <= kFzMaxPairs && d.E <= kFzMaxE &&
           d.k <= kFzMaxK && d.n_shared <= 4 && d.H % 256 == 0 && d.I / 128 <= kCombineMaxTiles;
}

// the two-pass path: activation records along H and along I, the unit table
// of the fused kernel's size
bool split_fits(const coli_moe_desc& d) {
    return d.E <= kFzMaxE && d.n_shared <= 4 && d.H % 256 == 0 && d.I % 256 == 0 &&
           d.H <= 256 * kActMaxGroups && d.I <= 256 * kActMaxGroups;
}

// with_fused: also the fused path's buffers (placed last, so the plan without
// them is a prefix of the plan with them)
WsPlan plan_ws(const coli_moe_desc& d, int T, int kind = kPlanFull) {
    WsPlan p;
    int64_t off = 0;
    auto take = [&](int64_t bytes) { const int64_t at = off; off = align256(off + bytes); return at; };
    const int64_t Tk = (int64_t)T * d.k;
    const int64_t P = (int64_t)T * (d.k + d.n_shared);
    p.zpart = take((int64_t)kMaxKS * T * d.E * 4);
    p.idx = take(Tk * 4);
    p.w = take(Tk * 4);
    p.offsets = take((int64_t)(d.E + 1) * 4);
    p.pair_tok = take(P * 4);
    p.pair_slot = take(Tk * 4);
    p.uniq = take((int64_t)d.E * 4);
    p.n_uniq = take(4);
    p.inv = take(Tk * 4);
    p.unit_expert = take((int64_t)(d.E + d.n_shared) * 4);
    p.unit_begin = take((int64_t)(d.E + d.n_shared) * 4);
    p.unit_end = take((int64_t)(d.E + d.n_shared) * 4);
    p.n_units = take(4);
    p.counters = take((int64_t)(d.H / 64) * 4);
    p.err = take(4);
    p.xq = take((int64_t)T * d.H * 4);          // fp16 hi + lo
    p.xinv = take((int64_t)T * (d.H / 64) * 4);
    p.hq = take(P * d.I * 4);                   // fp16 hi + lo
    p.hinv = take(P * (d.I / 64) * 4);
    p.o = take(P * d.H * 4);
    p.xg = p.o;                                 // tensor-core path: gathered fp16 tokens (dead
                                                //   before the down pass writes o)
    p.hg = take(P * d.I * 2);                   //   fp16 h of every pair
    p.hmax = take(P * 4);                       //   per-pair max |h|
    p.hsc = take(P * 4);                        //   per-pair inverse scale of h
    p.xq8 = p.part = p.queue = p.sel = p.hrec = p.squeue = 0;
    if (kind == kPlanFull && fused_fits(d, T)) {
        p.xq8 = take((int64_t)T * (d.H / 256) * kActRec);
        p.part = take(P * (d.I / 128) * d.H * 4);
        p.queue = take(4);
        p.sel = take((int64_t)T * d.E * 4);
    } else if (kind != kPlanBase && split_fits(d)) {
        p.xq8 = take((int64_t)T * (d.H / 256) * kActRec);
        p.hrec = take(P * (d.I / 256) * kActRec);
        p.squeue = take(2 * 4);
    }
    p.total = off;
    return p;
}

template <typename T> T* at(void* ws, int64_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int tokens_ok(const coli_moe_desc& d, int T) {
    if (T < 1 || T > 8192) return fail(COLI_E_INVAL, "T=%d outside [1, 8192]", T);
    const int64_t words = (int64_t)d.E * ((T + 31) / 32);
    if (words > 24576)
        return fail(COLI_E_UNSUPPORTED, "E*ceil(T/32)=%lld exceeds 24576 (union bitmap)",
                    (long long)words);
    return COLI_OK;
}

// Raise a kernel's dynamic shared-memory limit to `bytes` (static + dynamic
// above 48 KB needs the opt-in).  The largest value set per (device, kernel) is
// remembered so that a forward normally makes no attribute call.
int set_smem(const void* fn, int bytes) {
    struct Entry { int dev; const void* fn; int bytes; };
    static std::mutex mu;
    static std::vector<Entry> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(COLI_E_CUDA, "smem attribute: no device");
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& en : done)
        if (en.dev == dev && en.fn == fn && en.bytes >= bytes) return COLI_OK;
    const cudaError_t e =
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return fail(COLI_E_CUDA, "smem attribute: %s", cudaGetErrorString(e));
    for (Entry& en : done)
        if (en.dev == dev && en.fn == fn) { en.bytes = bytes; return COLI_OK; }
    done.push_back({dev, fn, bytes});
    return COLI_OK;
}

// Launch as a programmatic dependent of the previous kernel in the stream: the
// kernel may start while that one finishes and waits (griddepcontrol.wait)
// before it reads what that one wrote.
template <typename... Args>
int launch_pdl(void (*kern)(Args...), dim3 grid, int threads, int smem, cudaStream_t st,
               const char* what, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) return fail(COLI_E_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return check_launch(what);
}

// Router logits into zpart ([*ks_out][T][E] K slices; the small-batch router
// sums its slices itself and reports one).  When xq is non-null the
// fp16 activation operand is produced as well (by extra CTAs of the small-batch
// router, or by its own launch after the tiled router).
int launch_router(const coli_moe_desc& d, const void* x, coli_dtype xt, int T, float* zpart,
                  __half* xq, float* xinv, cudaStream_t st, int* ks_out,
                  const RouterExtras* fused = nullptr) {
    const bool row_ok = T <= kRouterRowMaxT && d.H <= kRouterRowMaxH && d.H % 4 == 0 &&
                        (reinterpret_cast<uintptr_t>(d.router_w) & 15) == 0;
    if (row_ok) {
        RouterExtras ex;
        if (fused) ex = *fused;
        ex.xq = xq;
        ex.xinv = xinv;
        const int qblocks = (ex.xq || ex.xq8) ? T : 0;
        const int zblocks = ex.zero_n > 0 ? 1 : 0;
        const dim3 grid(d.E + qblocks + zblocks);
        *ks_out = 1;
        if (xt == COLI_F32)
            return launch_pdl(router_row_kernel<float>, grid, 256, 0, st, "router", (const float*)x,
                              T, d.H, d.router_w, d.E, zpart, ex);
        return launch_pdl(router_row_kernel<__nv_bfloat16>, grid, 256, 0, st, "router",
                          (const __nv_bfloat16*)x, T, d.H, d.router_w, d.E, zpart, ex);
    }
    int KS = 0;
    if (T <= kRouterMaxT)
        for (int c : {8, 4, 2, 1})
            if (d.H % (c * 128) == 0 && d.H / c <= kRouterMaxSlice) { KS = c; break; }
    if (KS > 0) {
        const int rblocks = (d.E * KS + 7) / 8;
        RouterExtras ex;
        if (fused) ex = *fused;
        ex.xq = xq;
        ex.xinv = xinv;
        const int qblocks = (ex.xq || ex.xq8) ? T : 0;
        const int zblocks = ex.zero_n > 0 ? 1 : 0;
        const dim3 grid(rblocks + qblocks + zblocks);
        *ks_out = 1;
        if (xt == COLI_F32)
            return launch_pdl(router_gemv_kernel<float>, grid, 256, 0, st, "router",
                              (const float*)x, T, d.H, d.router_w, d.E, KS, zpart, rblocks, ex);
        return launch_pdl(router_gemv_kernel<__nv_bfloat16>, grid, 256, 0, st, "router",
                          (const __nv_bfloat16*)x, T, d.H, d.router_w, d.E, KS, zpart, rblocks, ex);
    } else {
        const int tiles = ((T + 63) / 64) * ((d.E + 63) / 64);
        KS = 1;
        for (int c : {8, 4, 2, 1})
            if (d.H % (c * 16) == 0 && (tiles * c <= 2 * 148 || c == 1)) { KS = c; break; }
        const dim3 grid((T + 63) / 64, (d.E + 63) / 64, KS);
        if (xt == COLI_F32)
            router_tiled_kernel<float><<<grid, 256, 0, st>>>((const float*)x, T, d.H, d.router_w, d.E, KS, zpart);
        else
            router_tiled_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, T, d.H, d.router_w, d.E, KS, zpart);
        if (xq) {
            int rc = check_launch("router");
            if (rc) return rc;
            if (xt == COLI_F32)
                act_quant_kernel<float><<<T, 256, 0, st>>>((const float*)x, T, d.H, xq, xinv);
            else
                act_quant_kernel<__nv_bfloat16><<<T, 256, 0, st>>>((const __nv_bfloat16*)x, T, d.H, xq, xinv);
        }
    }
    *ks_out = KS;
    return check_launch("router");
}

int launch_topk(const coli_moe_desc& d, const PickFilter& f, const float* zpart, int KS, int T,
                int32_t* idx, float* w, cudaStream_t st) {
    const int smem = kTopkWarps * 2 * d.E * 4;
    topk_kernel<<<(T + kTopkWarps - 1) / kTopkWarps, 32 * kTopkWarps, smem, st>>>(
        zpart, KS, T, d.E, d.router_b, d.k, d.routed_scale, d.norm_topk, f, idx, w);
    return check_launch("topk");
}

int union_smem_bytes(int T, int E) {
    return (int)((int64_t)E * ((T + 31) / 32) * 4 + 3 * (int64_t)E * 4);
}

int launch_union(const int32_t* idx, int T, int k, int E, const UnionOut& o, cudaStream_t st) {
    const int smem = union_smem_bytes(T, E);
    int rc = set_smem((const void*)union_kernel, smem);
    if (rc) return rc;
    union_kernel<<<1, kUnionThreads, smem, st>>>(idx, T, k, E, o);
    return check_launch("union");
}

// top-k + union; one fused single-CTA launch for small batches
int launch_select(const coli_moe_desc& d, const PickFilter& f, const float* zpart, int KS, int T,
                  int32_t* idx, float* w, const UnionOut& o, cudaStream_t st) {
    if (T * d.E <= kSmallSelect && T <= kSmallSelect / 32) {
        const int smem = std::max(2 * T * d.E * 4, union_smem_bytes(T, d.E));
        int rc = set_smem((const void*)topk_union_kernel, smem);
        if (rc) return rc;
        topk_union_kernel<<<1, kUnionThreads, smem, st>>>(zpart, KS, T, d.E, d.router_b, d.k,
                                                          d.routed_scale, d.norm_topk, f, idx, w, o);
        return check_launch("topk+union");
    }
    int rc = launch_topk(d, f, zpart, KS, T, idx, w, st);
    if (rc) return rc;
    return launch_union(idx, T, d.k, d.E, o, st);
}

// ---------------------------------------------------------------------------
// tensor-core path
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// [rows][cols] fp16, boxes of 64 rows x 64 columns, 128-byte swizzle
int encode_b_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(COLI_E_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kGemmMaxN};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(COLI_E_CUDA, "tensor map encode failed (%d)", (int)r);
    return COLI_OK;
}

// xq8 of T tokens as [T] rows of H/256 activation records read as 32-bit
// words; boxes of one record (one gate/up stage) of every token, no swizzle
int encode_act_map(CUtensorMap* m, const void* xq8, int T, int H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(COLI_E_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[2] = {(cuuint64_t)(H / 256 * kActRec / 4), (cuuint64_t)T};
    const cuuint64_t strides[1] = {(cuuint64_t)(H / 256 * kActRec)};
    const cuuint32_t box[2] = {(cuuint32_t)(kActRec / 4), (cuuint32_t)T};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(xq8), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(COLI_E_CUDA, "activation tensor map encode failed (%d)", (int)r);
    return COLI_OK;
}

int gemm_grid() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
    }
    return sms;
}

template <typename Mark>
int launch_gemm(const coli_moe_layer* l, int T, void* ws, const WsPlan& p, cudaStream_t st,
                Mark&& mark) {
    const coli_moe_desc& d = l->run;
    const int P = T * (d.k + d.n_shared);
    int rc;
    {
        const int64_t n = (int64_t)P * (d.H / 8);
        gather_x_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            at<__half>(ws, p.xq), at<int32_t>(ws, p.pair_tok), P, d.H, at<__half>(ws, p.xg),
            at<uint32_t>(ws, p.hmax));
        if ((rc = check_launch("gather x"))) return rc;
    }
    if ((rc = set_smem((const void*)moe_gemm_kernel, kGemmSmem))) return rc;
    GemmArgs g;
    g.store = l->store;
    g.L = l->L;
    g.n_units = at<int32_t>(ws, p.n_units);
    g.unit_expert = at<int32_t>(ws, p.unit_expert);
    g.unit_begin = at<int32_t>(ws, p.unit_begin);
    g.unit_end = at<int32_t>(ws, p.unit_end);
    g.pair_tok = at<int32_t>(ws, p.pair_tok);
    g.group = d.group;
    g.hf = at<float>(ws, p.hq);
    g.hmax = at<uint32_t>(ws, p.hmax);
    g.o = at<float>(ws, p.o);
    g.err = at<int32_t>(ws, p.err);
    g.I = d.I; g.H = d.H;
    CUtensorMap xmap, hmap;
    if ((rc = encode_b_map(&xmap, at<__half>(ws, p.xg), P, d.H))) return rc;
    g.two = 1; g.K = d.H; g.R = d.I;
    g.act_inv = at<float>(ws, p.xinv);
    moe_gemm_kernel<<<gemm_grid(), kGemmThreads, kGemmSmem, st>>>(xmap, g);
    if ((rc = check_launch("gate/up gemm"))) return rc;
    if ((rc = mark(COLI_STAGE_DOWN))) return rc;
    {
        const int64_t n = (int64_t)P * d.I / 2;
        convert_h_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
            at<float>(ws, p.hq), at<uint32_t>(ws, p.hmax), P, d.I, at<__half>(ws, p.hg),
            at<float>(ws, p.hsc));
        if ((rc = check_launch("convert h"))) return rc;
    }
    if ((rc = encode_b_map(&hmap, at<__half>(ws, p.hg), P, d.I))) return rc;
    g.two = 0; g.K = d.I; g.R = d.H;
    g.act_inv = at<float>(ws, p.hsc);
    moe_gemm_kernel<<<gemm_grid(), kGemmThreads, kGemmSmem, st>>>(hmap, g);
    return check_launch("down gemm");
}

// tensor cores from this many tokens on (the GEMV path below)
constexpr int kGemmMinTokens = 48;
bool gemm_path_preferred(const coli_moe_desc&, int T) { return T >= kGemmMinTokens; }

// AUTO past the fused path's limits: the two-pass path up to kSplitMaxT tokens
// (GLM-5.2 prefill shapes on B200: 1.33 ms against the GEMM path's 3.93 ms at
// 128 tokens, 2.28 against 4.17 ms at 512; the GEMM path wins at 2048, 6.7
// against 8.1 ms, once units hold enough tokens to fill its 64-token tiles)
constexpr int kSplitMaxT = 1024;
coli_path large_batch_path(const coli_moe_desc& d, int bits, int T) {
    if (bits == 4 && split_fits(d) && T <= kSplitMaxT && T > kFzMaxT) return COLI_PATH_TWOPASS;
    return gemm_path_preferred(d, T) ? COLI_PATH_GEMM : COLI_PATH_GEMV;
}

template <int NT, bool GS>
int launch_gateup_t(const coli_moe_desc& d, int units_max, const GemvArgs& a, cudaStream_t st) {
    const int smem = gemv_ring_bytes<true, GS>() + gemv_act_bytes(a.tok_cap, d.H);
    int rc = set_smem((const void*)gateup_gemv_kernel<NT, GS>, smem);
    if (rc) return rc;
    gateup_gemv_kernel<NT, GS><<<units_max * (d.I / 64), kGemvThreads, smem, st>>>(a);
    return check_launch("gate/up gemv");
}

template <int NT, bool GS>
int launch_down_t(const coli_moe_desc& d, int units_max, const GemvArgs& a, cudaStream_t st) {
    const int smem = gemv_ring_bytes<false, GS>() + gemv_act_bytes(a.tok_cap, d.I);
    int rc = set_smem((const void*)down_gemv_kernel<NT, GS>, smem);
    if (rc) return rc;
    down_gemv_kernel<NT, GS><<<units_max * (d.H / 64) * kDownSplit, kGemvThreads, smem, st>>>(a);
    return check_launch("down gemv");
}

template <typename Mark>
int launch_gemv(const coli_moe_layer* l, int T, void* ws, const WsPlan& p, const float* residual,
                float* y, cudaStream_t st, Mark&& mark) {
    const coli_moe_desc& d = l->run;
    GemvArgs a;
    a.store = l->store;
    a.L = l->L;
    a.n_units = at<int32_t>(ws, p.n_units);
    a.unit_expert = at<int32_t>(ws, p.unit_expert);
    a.unit_begin = at<int32_t>(ws, p.unit_begin);
    a.unit_end = at<int32_t>(ws, p.unit_end);
    a.pair_tok = at<int32_t>(ws, p.pair_tok);
    a.xq = at<__half>(ws, p.xq);
    a.xinv = at<float>(ws, p.xinv);
    a.hq = at<__half>(ws, p.hq);
    a.hinv = at<float>(ws, p.hinv);
    a.o = at<float>(ws, p.o);
    a.counters = at<int32_t>(ws, p.counters);
    a.inv = at<int32_t>(ws, p.inv);
    a.w = at<float>(ws, p.w);
    a.residual = residual;
    a.y = y;
    a.err = at<int32_t>(ws, p.err);
    // tokens staged per pass: as many as the MMA tiles take, but ring + staging
    // must fit one CTA's shared memory for the longer reduction
    a.tok_cap = std::min(T <= 4 ? 4 : 8, T);
    while (a.tok_cap > 1 &&
           gemv_ring_bytes<true, true>() + gemv_act_bytes(a.tok_cap, std::max(d.H, d.I)) > kGemvSmemMax)
        --a.tok_cap;
    a.T = T; a.k = d.k; a.n_shared = d.n_shared;
    a.H = d.H; a.I = d.I; a.group = d.group;
    const int units_max = (int)std::min<int64_t>(d.E, (int64_t)T * d.k) + d.n_shared;
    const bool gs = d.group != 0;
    int rc = T <= 4 ? (gs ? launch_gateup_t<1, true>(d, units_max, a, st) : launch_gateup_t<1, false>(d, units_max, a, st))
                    : (gs ? launch_gateup_t<2, true>(d, units_max, a, st) : launch_gateup_t<2, false>(d, units_max, a, st));
    if (rc) return rc;
    if ((rc = mark(COLI_STAGE_DOWN))) return rc;
    return T <= 4 ? (gs ? launch_down_t<1, true>(d, units_max, a, st) : launch_down_t<1, false>(d, units_max, a, st))
                  : (gs ? launch_down_t<2, true>(d, units_max, a, st) : launch_down_t<2, false>(d, units_max, a, st));
}

// ---------------------------------------------------------------------------
// fused small-batch path
// ---------------------------------------------------------------------------
int sm_count() { return gemm_grid(); }

// ---------------------------------------------------------------------------
// two-pass path: x records, gate/up pass (h in f32), h records, down pass (o)
// ---------------------------------------------------------------------------
template <bool GS>
int launch_split_t(const SplitArgs& a, cudaStream_t st, const char* what) {
    const int smem = a.slots * a.slot_bytes;
    int rc = set_smem((const void*)moe_split_kernel<GS>, smem);
    if (rc) return rc;
    return launch_pdl(moe_split_kernel<GS>, dim3(sm_count()), kFzThreads, smem, st, what, a);
}

template <typename Mark>
int launch_split(const coli_moe_layer* l, const void* x, coli_dtype xt, int T, void* ws,
                 const WsPlan& p, cudaStream_t st, Mark&& mark) {
    const coli_moe_desc& d = l->run;
    const int P = T * (d.k + d.n_shared);
    int8_t* xrec = at<int8_t>(ws, p.xq8);
    int rc = xt == COLI_F32
        ? launch_pdl(act_records_kernel<float>, dim3(T), 256, 0, st, "x records",
                     (const float*)x, d.H, xrec)
        : launch_pdl(act_records_kernel<__nv_bfloat16>, dim3(T), 256, 0, st, "x records",
                     (const __nv_bfloat16*)x, d.H, xrec);
    if (rc) return rc;
    SplitArgs a;
    a.store = l->store;
    a.L = l->L;
    a.n_units = at<int32_t>(ws, p.n_units);
    a.unit_expert = at<int32_t>(ws, p.unit_expert);
    a.unit_begin = at<int32_t>(ws, p.unit_begin);
    a.unit_end = at<int32_t>(ws, p.unit_end);
    a.pair_tok = at<int32_t>(ws, p.pair_tok);
    a.err = at<int32_t>(ws, p.err);
    a.H = d.H; a.I = d.I;
    a.slot_bytes = (int)align256(kFzActOff + kFzChunk * kActRec);
    const int budget = 227 * 1024 - (int)sizeof(SplitShared) - 1024;
    a.slots = std::min(kSpSlots, budget / a.slot_bytes);
    if (a.slots < 2) return fail(COLI_E_UNSUPPORTED, "two-pass: ring does not fit");
    const bool gs = d.group != 0;
    float* hf = at<float>(ws, p.hq);                 // [P][I] f32
    int8_t* hrec = at<int8_t>(ws, p.hrec);
    a.act = xrec;
    a.out = hf;
    a.queue = at<int32_t>(ws, p.squeue);
    a.down = 0;
    if ((rc = gs ? launch_split_t<true>(a, st, "gate/up pass") : launch_split_t<false>(a, st, "gate/up pass")))
        return rc;
    if ((rc = mark(COLI_STAGE_DOWN))) return rc;
    if ((rc = launch_pdl(act_records_kernel<float>, dim3(P), 256, 0, st, "h records",
                         (const float*)hf, d.I, hrec)))
        return rc;
    a.act = hrec;
    a.out = at<float>(ws, p.o);                      // [P][H] f32
    a.queue = at<int32_t>(ws, p.squeue) + 1;
    a.down = 1;
    return gs ? launch_split_t<true>(a, st, "down pass") : launch_split_t<false>(a, st, "down pass");
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous one (router, then fused) finishes; it waits
// (griddepcontrol.wait) before reading what that kernel wrote.

template <int NT, bool GS, bool W8, bool TW>
int launch_fused_t(const CUtensorMap& xmap, const FusedArgs& a, cudaStream_t st) {
    const int smem = a.slots * a.slot_bytes;
    int rc = set_smem((const void*)moe_fused_kernel<NT, GS, W8, TW>, smem);
    if (rc) return rc;
    return launch_pdl(moe_fused_kernel<NT, GS, W8, TW>, dim3(sm_count()), kFzThreads, smem, st,
                      "fused moe", xmap, a);
}

template <bool W8, bool TW>
int launch_fused_w(int NT, bool gs, const CUtensorMap& xmap, const FusedArgs& a, cudaStream_t st) {
    switch (NT) {
        case 1: return gs ? launch_fused_t<1, true, W8, TW>(xmap, a, st) : launch_fused_t<1, false, W8, TW>(xmap, a, st);
        case 2: return gs ? launch_fused_t<2, true, W8, TW>(xmap, a, st) : launch_fused_t<2, false, W8, TW>(xmap, a, st);
        default: return gs ? launch_fused_t<4, true, W8, TW>(xmap, a, st) : launch_fused_t<4, false, W8, TW>(xmap, a, st);
    }
}

template <typename Mark>
int launch_fused(const coli_moe_layer* l, int T, void* ws, const WsPlan& p, int KS,
                 const float* residual, float* y, cudaStream_t st, Mark&& mark) {
    const coli_moe_desc& d = l->run;
    FusedArgs a;
    a.store = l->store;
    a.L = l->L;
    a.filter = l->filter;
    a.withhold = l->withhold;
    (void)KS;  // the small-batch router leaves one slice: the scores themselves
    a.score = at<float>(ws, p.zpart);
    a.sel = at<float>(ws, p.sel);
    a.routed_scale = d.routed_scale;
    a.norm_topk = d.norm_topk;
    a.xq8 = at<int8_t>(ws, p.xq8);
    a.part = at<float>(ws, p.part);
    a.queue = at<int32_t>(ws, p.queue);
    a.idx = at<int32_t>(ws, p.idx);
    a.w = at<float>(ws, p.w);
    a.inv = at<int32_t>(ws, p.inv);
    a.err = at<int32_t>(ws, p.err);
    a.T = T; a.E = d.E; a.k = d.k; a.n_shared = d.n_shared;
    a.H = d.H; a.I = d.I; a.group = d.group;
    const int NT = T <= 4 ? 1 : (T <= 8 ? 2 : 4);
    a.slot_bytes = (int)align256(kFzActOff + 4 * NT * kActRec);
    const int budget = 227 * 1024 - (int)sizeof(FusedShared) - 1024;
    a.slots = std::min(kFzSlots, budget / a.slot_bytes);
    if (a.slots < 2) return fail(COLI_E_UNSUPPORTED, "fused: ring does not fit");
    const bool gs = d.group != 0;
    int rc;
    // 2 to 4 tokens: one TMA box brings every token's activation slice of a stage
    CUtensorMap xmap;
    std::memset(&xmap, 0, sizeof(xmap));
    a.act_tma = 0;
    if (T >= 2 && NT == 1) {
        if ((rc = encode_act_map(&xmap, a.xq8, T, d.H))) return rc;
        a.act_tma = 1;
    }
    // the wait test has its own instantiation (4-bit layers only)
    if (l->withhold >= 0 && l->bits == 8)
        return fail(COLI_E_UNSUPPORTED, "wait test: 4-bit layers only");
    rc = l->bits == 8 ? launch_fused_w<true, false>(NT, gs, xmap, a, st)
                      : (l->withhold >= 0 ? launch_fused_w<false, true>(NT, gs, xmap, a, st)
                                          : launch_fused_w<false, false>(NT, gs, xmap, a, st));
    if (rc) return rc;
    if ((rc = mark(COLI_STAGE_DOWN))) return rc;
    if ((rc = mark(COLI_STAGE_COMBINE))) return rc;
    CombineArgs c;
    c.part = a.part;
    c.w = a.w;
    c.inv = a.inv;
    c.residual = residual;
    c.y = y;
    c.T = T; c.k = d.k; c.n_shared = d.n_shared; c.H = d.H; c.TG = d.I / 128;
    const int warps = std::min(32, d.k + d.n_shared);
    return launch_pdl(moe_combine_kernel, dim3(T * (d.H / 32)), 32 * warps, 0, st, "fused combine", c);
}

}  // namespace

// ---------------------------------------------------------------------------
// Allocation-free forward: the workspace is a scratch array compiled into the
// library (one copy per device), not memory from the caller.
// ---------------------------------------------------------------------------
namespace {
__device__ __align__(256) unsigned char g_noalloc_scratch[COLI_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoallocEntry { void* ctx; void* ptr; };
NoallocEntry g_noalloc[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(f);
    });
    return fn;
}

// Device address of this device's copy of the scratch array.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the device current, once per device and context: a context created anew
// (after cudaDeviceReset, or after the primary context was released) loads the
// module again, possibly at another address, so the lookup is repeated then.
int noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return fail(COLI_E_CUDA, "forward_noalloc: no usable current device");
    CtxGetCurrentFn get = ctx_get_current_fn();
    if (!get) return fail(COLI_E_CUDA, "forward_noalloc: cuCtxGetCurrent is not available");
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocEntry& en = g_noalloc[dev];
    if (!ctx || en.ctx != (void*)ctx || !en.ptr) {
        // the lookup also makes the device's primary context current if the
        // runtime had not created it yet
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(COLI_E_CUDA, "forward_noalloc: scratch lookup failed: %s",
                        cudaGetErrorString(e));
        if (get(&ctx) != CUDA_SUCCESS || !ctx)
            return fail(COLI_E_CUDA, "forward_noalloc: no current context on device %d", dev);
        en.ctx = (void*)ctx;
        en.ptr = p;
    }
    *out = en.ptr;
    return COLI_OK;
}
}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* coli_moe_last_error(void) { return g_err.c_str(); }

int coli_moe_quantize(const float* w, int64_t rows, int64_t cols, int32_t group,
                      uint8_t* packed, float* scales) {
    if (!w || !packed || !scales) return fail(COLI_E_INVAL, "quantize: NULL pointer");
    if (rows < 0 || cols <= 0 || cols % 2 || (group != 0 && group != 64) ||
        (group && cols % group))
        return fail(COLI_E_INVAL, "quantize: bad shape rows=%lld cols=%lld group=%d",
                    (long long)rows, (long long)cols, group);
    const int64_t gs = group ? group : cols, ng = cols / gs;
    for (int64_t r = 0; r < rows; ++r) {
        const float* row = w + r * cols;
        uint8_t* prow = packed + r * (cols / 2);
        for (int64_t g = 0; g < ng; ++g) {
            float m = 0.0f;
            for (int64_t c = g * gs; c < (g + 1) * gs; ++c) m = std::fmax(m, std::fabs(row[c]));
            const float s = m / 7.0f;
            scales[r * ng + g] = s;
            for (int64_t c = g * gs; c < (g + 1) * gs; c += 2) {
                int q[2];
                for (int i = 0; i < 2; ++i) {
                    float v = s == 0.0f ? 0.0f : std::rint(row[c + i] / s);
                    v = std::fmin(std::fmax(v, -7.0f), 7.0f);
                    q[i] = (int)v;
                }
                prow[c / 2] = (uint8_t)((q[0] & 15) | ((q[1] & 15) << 4));
            }
        }
    }
    return COLI_OK;
}

int coli_moe_expert_bytes(int32_t H, int32_t I, int32_t group, size_t* bytes) {
    if (!bytes) return fail(COLI_E_INVAL, "expert_bytes: NULL pointer");
    if (!shape_ok(H, I, group)) return fail(COLI_E_INVAL, "expert_bytes: bad shape");
    *bytes = (size_t)make_blob_layout(H, I, group).bytes;
    return COLI_OK;
}

int coli_moe_pack_expert(int32_t H, int32_t I, int32_t group, const uint8_t* gate_codes,
                         const float* gate_scales, const uint8_t* up_codes,
                         const float* up_scales, const uint8_t* down_codes,
                         const float* down_scales, void* blob) {
    if (!gate_codes || !gate_scales || !up_codes || !up_scales || !down_codes ||
        !down_scales || !blob)
        return fail(COLI_E_INVAL, "pack_expert: NULL pointer");
    if (!shape_ok(H, I, group)) return fail(COLI_E_INVAL, "pack_expert: bad shape");
    const BlobLayout L = make_blob_layout(H, I, group);
    uint8_t* out = static_cast<uint8_t*>(blob);
    std::memset(out, 0, (size_t)L.bytes);
    const uint8_t* codes[3] = {gate_codes, up_codes, down_codes};
    const float* scales[3] = {gate_scales, up_scales, down_scales};
    for (int m = 0; m < 3; ++m) {
        const int R = L.rows[m], K = L.cols[m], ng = L.ngroups[m];
        for (int r = 0; r < R; ++r) {
            for (int c = 0; c < K; ++c) {
                const uint8_t byte = codes[m][(int64_t)r * (K / 2) + c / 2];
                const uint32_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
                uint32_t* word = reinterpret_cast<uint32_t*>(out + L.codes[m] + frag_word_offset(r, c, K));
                *word |= nib << frag_nibble_shift(r, c);
            }
            for (int g = 0; g < ng; ++g)
                reinterpret_cast<float*>(out + L.scales[m])[scale_offset(r, g, ng)] =
                    scales[m][(int64_t)r * ng + g];
        }
    }
    return COLI_OK;
}

int coli_moe_quantize8(const float* w, int64_t rows, int64_t cols, int32_t group, int8_t* codes,
                       float* scales) {
    if (!w || !codes || !scales) return fail(COLI_E_INVAL, "quantize8: NULL pointer");
    if (rows < 0 || cols <= 0 || (group != 0 && group != 64) || (group && cols % group))
        return fail(COLI_E_INVAL, "quantize8: bad shape rows=%lld cols=%lld group=%d",
                    (long long)rows, (long long)cols, group);
    const int64_t gs = group ? group : cols, ng = cols / gs;
    for (int64_t r = 0; r < rows; ++r) {
        const float* row = w + r * cols;
        for (int64_t g = 0; g < ng; ++g) {
            float m = 0.0f;
            for (int64_t c = g * gs; c < (g + 1) * gs; ++c) m = std::fmax(m, std::fabs(row[c]));
            const float s = m / 127.0f;
            scales[r * ng + g] = s;
            for (int64_t c = g * gs; c < (g + 1) * gs; ++c) {
                int q = 0;
                if (s != 0.0f) q = (int)std::fmin(std::fmax(std::rint(row[c] / s), -127.0f), 127.0f);
                codes[r * cols + c] = (int8_t)q;
            }
        }
    }
    return COLI_OK;
}

int coli_moe_expert_bytes8(int32_t H, int32_t I, int32_t group, size_t* bytes) {
    if (!bytes) return fail(COLI_E_INVAL, "expert_bytes8: NULL pointer");
    if (!shape_ok(H, I, group)) return fail(COLI_E_INVAL, "expert_bytes8: bad shape");
    *bytes = (size_t)make_blob_layout8(H, I, group).bytes;
    return COLI_OK;
}

int coli_moe_pack_expert8(int32_t H, int32_t I, int32_t group, const int8_t* gate_codes,
                          const float* gate_scales, const int8_t* up_codes, const float* up_scales,
                          const int8_t* down_codes, const float* down_scales, void* blob) {
    if (!gate_codes || !gate_scales || !up_codes || !up_scales || !down_codes || !down_scales ||
        !blob)
        return fail(COLI_E_INVAL, "pack_expert8: NULL pointer");
    if (!shape_ok(H, I, group)) return fail(COLI_E_INVAL, "pack_expert8: bad shape");
    const BlobLayout L = make_blob_layout8(H, I, group);
    uint8_t* out = static_cast<uint8_t*>(blob);
    std::memset(out, 0, (size_t)L.bytes);
    const int8_t* codes[3] = {gate_codes, up_codes, down_codes};
    const float* scales[3] = {gate_scales, up_scales, down_scales};
    for (int m = 0; m < 3; ++m) {
        const int R = L.rows[m], K = L.cols[m], ng = L.ngroups[m];
        for (int r = 0; r < R; ++r) {
            for (int c = 0; c < K; ++c)
                out[L.codes[m] + frag8_byte_offset(r, c, K)] =
                    (uint8_t)codes[m][(int64_t)r * K + c];
            for (int g = 0; g < ng; ++g)
                reinterpret_cast<float*>(out + L.scales[m])[scale_offset(r, g, ng)] =
                    scales[m][(int64_t)r * ng + g];
        }
    }
    return COLI_OK;
}

int coli_moe_quantize_expert_device(int32_t H, int32_t I, int32_t group, const float* gate,
                                    const float* up, const float* down, void* blob,
                                    coli_stream_t stream) {
    if (!gate || !up || !down || !blob) return fail(COLI_E_INVAL, "quantize_expert_device: NULL pointer");
    if (!shape_ok(H, I, group)) return fail(COLI_E_INVAL, "quantize_expert_device: bad shape");
    const BlobLayout L = make_blob_layout(H, I, group);
    uint8_t* b = static_cast<uint8_t*>(blob);
    const float* src[3] = {gate, up, down};
    for (int m = 0; m < 3; ++m) {
        const int R = L.rows[m], K = L.cols[m];
        const int smem = 16 * (K / 2);
        int rc = set_smem((const void*)quantize_rows_kernel<QzF32>, smem);
        if (rc) return rc;
        quantize_rows_kernel<<<R / 16, 256, smem, S(stream)>>>(
            QzF32{src[m]}, R, K, group, b + L.codes[m], reinterpret_cast<float*>(b + L.scales[m]));
        if ((rc = check_launch("quantize_rows"))) return rc;
    }
    return COLI_OK;
}

int coli_moe_quantize_expert8_device(int32_t H, int32_t I, int32_t group, const float* gate,
                                     const float* up, const float* down, void* blob,
                                     coli_stream_t stream) {
    if (!gate || !up || !down || !blob) return fail(COLI_E_INVAL, "quantize_expert8_device: NULL pointer");
    if (!shape_ok(H, I, group)) return fail(COLI_E_INVAL, "quantize_expert8_device: bad shape");
    const BlobLayout L = make_blob_layout8(H, I, group);
    uint8_t* b = static_cast<uint8_t*>(blob);
    const float* src[3] = {gate, up, down};
    for (int m = 0; m < 3; ++m) {
        const int R = L.rows[m], K = L.cols[m];
        const int smem = 16 * K;
        int rc = set_smem((const void*)quantize_rows8_kernel<QzF32>, smem);
        if (rc) return rc;
        quantize_rows8_kernel<<<R / 16, 256, smem, S(stream)>>>(
            QzF32{src[m]}, R, K, group, b + L.codes[m], reinterpret_cast<float*>(b + L.scales[m]));
        if ((rc = check_launch("quantize_rows8"))) return rc;
    }
    return COLI_OK;
}

int coli_moe_quantize_expert_fp8_device(int32_t H, int32_t I, int32_t group, const uint8_t* gate,
                                        const uint8_t* up, const uint8_t* down, const float* gate_bs,
                                        const float* up_bs, const float* down_bs, void* blob,
                                        coli_stream_t stream) {
    if (!gate || !up || !down || !gate_bs || !up_bs || !down_bs || !blob)
        return fail(COLI_E_INVAL, "quantize_expert_fp8_device: NULL pointer");
    if (!shape_ok(H, I, group)) return fail(COLI_E_INVAL, "quantize_expert_fp8_device: bad shape");
    const BlobLayout L = make_blob_layout(H, I, group);
    uint8_t* b = static_cast<uint8_t*>(blob);
    const uint8_t* src[3] = {gate, up, down};
    const float* bsrc[3] = {gate_bs, up_bs, down_bs};
    for (int m = 0; m < 3; ++m) {
        const int R = L.rows[m], K = L.cols[m];
        const int smem = 16 * (K / 2);
        int rc = set_smem((const void*)quantize_rows_kernel<QzFp8Block>, smem);
        if (rc) return rc;
        quantize_rows_kernel<<<R / 16, 256, smem, S(stream)>>>(
            QzFp8Block{src[m], bsrc[m], (K + 127) / 128}, R, K, group, b + L.codes[m],
            reinterpret_cast<float*>(b + L.scales[m]));
        if ((rc = check_launch("quantize_rows_fp8"))) return rc;
    }
    return COLI_OK;
}

int coli_moe_layer_create(const coli_moe_desc* desc, coli_moe_layer** out) {
    if (!desc || !out) return fail(COLI_E_INVAL, "layer_create: NULL pointer");
    const coli_moe_desc& d = *desc;
    if (!shape_ok(d.H, d.I, d.group)) return fail(COLI_E_INVAL, "layer_create: H, I must be multiples of 128, group 0 or 64");
    if (d.E < 1 || d.E > 1024 || d.k < 1 || d.k > 32 || d.k > d.E || d.n_shared < 0 || d.n_shared > 4)
        return fail(COLI_E_INVAL, "layer_create: need 1<=k<=min(E,32), E<=1024, 0<=n_shared<=4");
    if (!d.router_w || !d.router_b || !d.experts) return fail(COLI_E_INVAL, "layer_create: NULL device pointer");
    if (!(std::isfinite(d.routed_scale))) return fail(COLI_E_INVAL, "layer_create: routed_scale not finite");
    if (d.bits != 0 && d.bits != 4 && d.bits != 8)
        return fail(COLI_E_INVAL, "layer_create: bits must be 0 (4), 4 or 8, got %d", d.bits);
    coli_moe_layer* l = new (std::nothrow) coli_moe_layer;
    if (!l) return fail(COLI_E_NOMEM, "layer_create: out of host memory");
    l->d = d;
    l->bits = d.bits == 8 ? 8 : 4;
    l->L = l->bits == 8 ? make_blob_layout8(d.H, d.I, d.group) : make_blob_layout(d.H, d.I, d.group);
    l->run = d;
    const uint8_t* base = static_cast<const uint8_t*>(d.experts);
    l->store = ExpertStore{base, base + (int64_t)d.E * l->L.bytes, l->L.bytes, 0, d.E};
    l->filter = PickFilter{};
    l->filter.e_hi = d.E;
    *out = l;
    return COLI_OK;
}

int coli_moe_layer_set_wait_test(coli_moe_layer* layer, int32_t withhold_stage) {
    if (!layer) return fail(COLI_E_INVAL, "set_wait_test: NULL layer");
    layer->withhold = withhold_stage < 0 ? -1 : withhold_stage;
    return COLI_OK;
}

int coli_moe_layer_set_topp(coli_moe_layer* layer, float p) {
    if (!layer) return fail(COLI_E_INVAL, "set_topp: NULL layer");
    if (!(p >= 0.0f && p <= 1.0f)) return fail(COLI_E_INVAL, "set_topp: p=%g outside [0, 1]", (double)p);
    layer->filter.topp = p;
    return COLI_OK;
}

int coli_moe_layer_set_partition(coli_moe_layer* layer, int32_t e_begin, int32_t e_end,
                                 int32_t with_shared, const void* experts) {
    if (!layer || !experts) return fail(COLI_E_INVAL, "set_partition: NULL pointer");
    const coli_moe_desc& d = layer->d;
    if (e_begin < 0 || e_end < e_begin || e_end > d.E)
        return fail(COLI_E_INVAL, "set_partition: range [%d, %d) outside [0, %d)", e_begin, e_end, d.E);
    const uint8_t* base = static_cast<const uint8_t*>(experts);
    layer->run = d;
    layer->run.experts = experts;
    layer->run.n_shared = with_shared ? d.n_shared : 0;
    layer->store = ExpertStore{base, base + (int64_t)(e_end - e_begin) * layer->L.bytes,
                               layer->L.bytes, e_begin, d.E};
    layer->filter.e_lo = e_begin;
    layer->filter.e_hi = e_end;
    return COLI_OK;
}

int coli_moe_layer_destroy(coli_moe_layer* layer) {
    delete layer;
    return COLI_OK;
}

int coli_moe_workspace_size(const coli_moe_layer* layer, int32_t T, size_t* bytes) {
    if (!layer || !bytes) return fail(COLI_E_INVAL, "workspace_size: NULL pointer");
    int rc = tokens_ok(layer->run, T);
    if (rc) return rc;
    *bytes = (size_t)plan_ws(layer->run, T).total;
    return COLI_OK;
}

int coli_moe_route(const coli_moe_layer* layer, const void* x, coli_dtype xt, int32_t T,
                   int32_t* idx, float* w, void* ws, size_t ws_bytes, coli_stream_t stream) {
    if (!layer || !x || !idx || !w) return fail(COLI_E_INVAL, "route: NULL pointer");
    if (xt != COLI_F32 && xt != COLI_BF16) return fail(COLI_E_INVAL, "route: bad dtype");
    int rc = tokens_ok(layer->run, T);
    if (rc) return rc;
    const WsPlan p = plan_ws(layer->run, T);
    if (!ws || ws_bytes < (size_t)p.total)
        return fail(COLI_E_WORKSPACE, "route: workspace %zu < %lld bytes", ws_bytes, (long long)p.total);
    int KS;
    if ((rc = launch_router(layer->d, x, xt, T, at<float>(ws, p.zpart), nullptr, nullptr,
                            S(stream), &KS)))
        return rc;
    return launch_topk(layer->d, PickFilter{}, at<float>(ws, p.zpart), KS, T, idx, w, S(stream));
}

int coli_moe_union(const int32_t* idx, int32_t T, int32_t k, int32_t E, int32_t* offsets,
                   int32_t* pair_tok, int32_t* pair_slot, int32_t* uniq, int32_t* n_uniq,
                   coli_stream_t stream) {
    if (!idx || !offsets || !pair_tok || !pair_slot || !uniq || !n_uniq)
        return fail(COLI_E_INVAL, "union: NULL pointer");
    if (E < 1 || E > 1024 || k < 1 || k > 32 || T < 1 || T > 8192)
        return fail(COLI_E_INVAL, "union: bad sizes T=%d k=%d E=%d", T, k, E);
    if ((int64_t)E * ((T + 31) / 32) > 24576) return fail(COLI_E_UNSUPPORTED, "union: E*ceil(T/32) > 24576");
    UnionOut o{};
    o.offsets = offsets; o.pair_tok = pair_tok; o.pair_slot = pair_slot;
    o.uniq = uniq; o.n_uniq = n_uniq;
    return launch_union(idx, T, k, E, o, S(stream));
}

int coli_moe_forward_ex(const coli_moe_layer* layer, const void* x, coli_dtype xt, int32_t T,
                        float* y, const float* residual, coli_path path, int32_t* idx_out,
                        float* w_out, void* const* events, void* ws, size_t ws_bytes,
                        coli_stream_t stream) {
    if (!layer || !x || !y) return fail(COLI_E_INVAL, "forward: NULL pointer");
    if (xt != COLI_F32 && xt != COLI_BF16) return fail(COLI_E_INVAL, "forward: bad dtype");
    if (path != COLI_PATH_AUTO && path != COLI_PATH_GEMV && path != COLI_PATH_GEMM &&
        path != COLI_PATH_FUSED && path != COLI_PATH_TWOPASS)
        return fail(COLI_E_INVAL, "forward: bad path");
    const coli_moe_desc& d = layer->run;
    int rc = tokens_ok(d, T);
    if (rc) return rc;
    if (path == COLI_PATH_FUSED && !fused_fits(d, T))
        return fail(COLI_E_UNSUPPORTED,
                    "forward: fused path needs T<=%d, T*(k+n_shared)<=%d, E<=%d, k<=%d, n_shared<=4, "
                    "H%%256==0, I<=4096", kFzMaxT, kFzMaxPairs, kFzMaxE, kFzMaxK);
    if (path == COLI_PATH_TWOPASS && !split_fits(d))
        return fail(COLI_E_UNSUPPORTED, "forward: two-pass path needs E<=%d, n_shared<=4, "
                    "H%%256==0, I%%256==0", kFzMaxE);
    if (layer->bits == 8 && (path == COLI_PATH_GEMV || path == COLI_PATH_GEMM ||
                             path == COLI_PATH_TWOPASS ||
                             (path == COLI_PATH_AUTO && !fused_fits(d, T))))
        return fail(COLI_E_UNSUPPORTED, "forward: 8-bit experts run on the fused path only (T<=%d, "
                    "T*(k+n_shared)<=%d, E<=%d, H%%256==0, I<=4096)", kFzMaxT, kFzMaxPairs, kFzMaxE);
    if (path == COLI_PATH_AUTO)
        path = fused_fits(d, T) ? COLI_PATH_FUSED : large_batch_path(d, layer->bits, T);
    // the GEMV and GEMM paths need only a prefix of the full workspace
    const WsPlan p = plan_ws(d, T, path == COLI_PATH_FUSED ? kPlanFull
                                   : (path == COLI_PATH_TWOPASS ? kPlanSplit : kPlanBase));
    if (!ws || ws_bytes < (size_t)p.total)
        return fail(COLI_E_WORKSPACE, "forward: workspace %zu < %lld bytes", ws_bytes, (long long)p.total);
    cudaStream_t st = S(stream);
    int32_t* idx = at<int32_t>(ws, p.idx);
    float* w = at<float>(ws, p.w);
    auto mark = [&](int s) -> int {
        if (!events || !events[s]) return COLI_OK;
        // External: inside stream capture the record becomes an event node of the graph
        if (cudaEventRecordWithFlags(reinterpret_cast<cudaEvent_t>(events[s]), st,
                                     cudaEventRecordExternal) != cudaSuccess)
            return fail(COLI_E_CUDA, "forward: event record failed");
        return COLI_OK;
    };
    const bool gemm = path == COLI_PATH_GEMM;
    int KS;
    if (path == COLI_PATH_FUSED) {
        if ((rc = mark(COLI_STAGE_ROUTER))) return rc;
        RouterExtras ex;
        ex.xq8 = at<int8_t>(ws, p.xq8);
        ex.zero = at<int32_t>(ws, p.queue);
        ex.zero_n = 1;
        ex.err = at<int32_t>(ws, p.err);
        ex.sel = at<float>(ws, p.sel);
        ex.bias = d.router_b;
        if ((rc = launch_router(d, x, xt, T, at<float>(ws, p.zpart), nullptr, nullptr, st, &KS, &ex)))
            return rc;
        // the fused kernel is the union, gate/up and down stages at once
        if ((rc = mark(COLI_STAGE_UNION))) return rc;
        if ((rc = mark(COLI_STAGE_GATEUP))) return rc;
        if ((rc = launch_fused(layer, T, ws, p, KS, residual, y, st, mark))) return rc;
        if ((rc = mark(COLI_STAGES))) return rc;
        if (idx_out && cudaMemcpyAsync(idx_out, idx, sizeof(int32_t) * T * d.k,
                                       cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return fail(COLI_E_CUDA, "forward: copy idx");
        if (w_out && cudaMemcpyAsync(w_out, w, sizeof(float) * T * d.k,
                                     cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return fail(COLI_E_CUDA, "forward: copy w");
        return COLI_OK;
    }
    if ((rc = mark(COLI_STAGE_ROUTER))) return rc;
    const bool split = path == COLI_PATH_TWOPASS;
    // the two-pass path makes its own activation records after the union
    if ((rc = launch_router(d, x, xt, T, at<float>(ws, p.zpart), split ? nullptr : at<__half>(ws, p.xq),
                            split ? nullptr : at<float>(ws, p.xinv), st, &KS)))
        return rc;
    UnionOut o{};
    o.offsets = at<int32_t>(ws, p.offsets);
    o.pair_tok = at<int32_t>(ws, p.pair_tok);
    o.pair_slot = at<int32_t>(ws, p.pair_slot);
    o.uniq = at<int32_t>(ws, p.uniq);
    o.n_uniq = at<int32_t>(ws, p.n_uniq);
    o.inv = at<int32_t>(ws, p.inv);
    o.unit_expert = at<int32_t>(ws, p.unit_expert);
    o.unit_begin = at<int32_t>(ws, p.unit_begin);
    o.unit_end = at<int32_t>(ws, p.unit_end);
    o.n_units = at<int32_t>(ws, p.n_units);
    o.counters = at<int32_t>(ws, split ? p.squeue : p.counters);
    o.n_counters = split ? 2 : d.H / 64;
    o.err = at<int32_t>(ws, p.err);
    o.n_shared = d.n_shared;
    o.w = w;  // picks of weight 0 (not computed by this call) are left out
    if ((rc = mark(COLI_STAGE_UNION))) return rc;
    if ((rc = launch_select(d, layer->filter, at<float>(ws, p.zpart), KS, T, idx, w, o, st)))
        return rc;
    if ((rc = mark(COLI_STAGE_GATEUP))) return rc;
    if (gemm || split) {
        if ((rc = split ? launch_split(layer, x, xt, T, ws, p, st, mark)
                        : launch_gemm(layer, T, ws, p, st, mark)))
            return rc;
        if ((rc = mark(COLI_STAGE_COMBINE))) return rc;
        const int64_t n4 = (int64_t)T * (d.H / 4);
        combine_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(
            at<float>(ws, p.o), at<int32_t>(ws, p.inv), at<float>(ws, p.w), T, d.k, d.n_shared,
            d.H, residual, y);
        if ((rc = check_launch("combine"))) return rc;
    } else {
        if ((rc = launch_gemv(layer, T, ws, p, residual, y, st, mark))) return rc;
        if ((rc = mark(COLI_STAGE_COMBINE))) return rc;   // combine is fused into the down pass
    }
    if ((rc = mark(COLI_STAGES))) return rc;
    if (idx_out) {
        if (cudaMemcpyAsync(idx_out, idx, sizeof(int32_t) * T * d.k, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return fail(COLI_E_CUDA, "forward: copy idx");
    }
    if (w_out) {
        if (cudaMemcpyAsync(w_out, w, sizeof(float) * T * d.k, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return fail(COLI_E_CUDA, "forward: copy w");
    }
    return COLI_OK;
}

int coli_moe_forward(const coli_moe_layer* layer, const void* x, coli_dtype xt, int32_t T,
                     float* y, void* ws, size_t ws_bytes, coli_stream_t stream) {
    return coli_moe_forward_ex(layer, x, xt, T, y, nullptr, COLI_PATH_AUTO, nullptr, nullptr,
                               nullptr, ws, ws_bytes, stream);
}

int coli_moe_rmsnorm(const float* x, int32_t T, int32_t H, float eps, float* out,
                     coli_stream_t stream) {
    if (!x || !out) return fail(COLI_E_INVAL, "rmsnorm: NULL pointer");
    if (T < 1 || H < 4 || H % 4) return fail(COLI_E_INVAL, "rmsnorm: bad shape");
    return launch_pdl(rmsnorm_kernel, dim3(T), 256, 0, S(stream), "rmsnorm", x, (int)H, eps, out);
}

int coli_moe_stack_workspace_size(const coli_moe_layer* const* layers, int32_t L, int32_t T,
                                  size_t* bytes) {
    if (!layers || !bytes || L < 1) return fail(COLI_E_INVAL, "stack_workspace_size: bad arguments");
    size_t mx = 0;
    for (int l = 0; l < L; ++l) {
        if (!layers[l]) return fail(COLI_E_INVAL, "stack: NULL layer");
        size_t b;
        int rc = coli_moe_workspace_size(layers[l], T, &b);
        if (rc) return rc;
        mx = std::max(mx, b);
        if (layers[l]->d.H != layers[0]->d.H) return fail(COLI_E_INVAL, "stack: layers differ in H");
    }
    *bytes = (size_t)align256((int64_t)mx) + (size_t)T * layers[0]->d.H * 4;
    return COLI_OK;
}

int coli_moe_stack_forward(const coli_moe_layer* const* layers, int32_t L, float* x, int32_t T,
                           float eps, coli_path path, void* ws, size_t ws_bytes,
                           coli_stream_t stream) {
    size_t need;
    int rc = coli_moe_stack_workspace_size(layers, L, T, &need);
    if (rc) return rc;
    if (!x) return fail(COLI_E_INVAL, "stack_forward: NULL x");
    if (!ws || ws_bytes < need) return fail(COLI_E_WORKSPACE, "stack_forward: workspace %zu < %zu", ws_bytes, need);
    const int H = layers[0]->d.H;
    const size_t layer_ws = need - (size_t)T * H * 4;
    float* xn = reinterpret_cast<float*>(static_cast<char*>(ws) + layer_ws);
    for (int l = 0; l < L; ++l) {
        if ((rc = coli_moe_rmsnorm(x, T, H, eps, xn, stream))) return rc;
        if ((rc = coli_moe_forward_ex(layers[l], xn, COLI_F32, T, x, x, path, nullptr, nullptr,
                                      nullptr, ws, layer_ws, stream)))
            return rc;
    }
    return COLI_OK;
}

// ---------------------------------------------------------------------------
// Host-buffer entry points: x is copied into staging at the end of the
// workspace, the device forward runs, y is copied back; all on one stream.
// Page-locked memory that is mapped into the device's address space (what
// cudaHostAlloc gives on a unified-address system) is copied by a small
// kernel; anything else by cudaMemcpyAsync.
// ---------------------------------------------------------------------------
namespace {
int stage_copy(const void* src, void* dst, size_t bytes, bool h2d, cudaStream_t st) {
    void* mapped = nullptr;
    const void* host = h2d ? src : dst;
    if (bytes % 4 == 0 &&
        cudaHostGetDevicePointer(&mapped, const_cast<void*>(host), 0) == cudaSuccess && mapped) {
        const int64_t words = (int64_t)(bytes / 16) + 1;
        const int grid = (int)std::min<int64_t>(4 * sm_count(), (words + 255) / 256);
        stage_copy_kernel<<<grid, 256, 0, st>>>(h2d ? mapped : src, h2d ? dst : mapped,
                                                (int64_t)bytes);
        return check_launch(h2d ? "stage in" : "stage out");
    }
    (void)cudaGetLastError();  // not mapped: clear the query's error, copy by DMA
    if (cudaMemcpyAsync(dst, src, bytes, h2d ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost,
                        st) != cudaSuccess)
        return fail(COLI_E_CUDA, "host copy failed");
    return COLI_OK;
}
}  // namespace

int coli_moe_host_workspace_size(const coli_moe_layer* layer, int32_t T, size_t* bytes) {
    size_t b;
    int rc = coli_moe_workspace_size(layer, T, &b);
    if (rc) return rc;
    const int64_t row = (int64_t)T * layer->d.H * 4;
    *bytes = (size_t)(align256((int64_t)b) + 2 * align256(row));
    return COLI_OK;
}

int coli_moe_forward_host(const coli_moe_layer* layer, const void* x_host, coli_dtype xt,
                          int32_t T, float* y_host, coli_path path, void* ws, size_t ws_bytes,
                          coli_stream_t stream) {
    if (!layer || !x_host || !y_host) return fail(COLI_E_INVAL, "forward_host: NULL pointer");
    if (xt != COLI_F32 && xt != COLI_BF16) return fail(COLI_E_INVAL, "forward_host: bad dtype");
    size_t need, inner;
    int rc = coli_moe_host_workspace_size(layer, T, &need);
    if (rc) return rc;
    if ((rc = coli_moe_workspace_size(layer, T, &inner))) return rc;
    if (!ws || ws_bytes < need)
        return fail(COLI_E_WORKSPACE, "forward_host: workspace %zu < %zu bytes", ws_bytes, need);
    const int64_t row = (int64_t)T * layer->d.H * 4;
    char* base = static_cast<char*>(ws);
    void* xd = base + align256((int64_t)inner);
    float* yd = reinterpret_cast<float*>(base + align256((int64_t)inner) + align256(row));
    const size_t xbytes = (size_t)T * layer->d.H * (xt == COLI_F32 ? 4 : 2);
    if ((rc = stage_copy(x_host, xd, xbytes, true, S(stream)))) return rc;
    // y mapped into the device's address space: the layer's last kernel writes
    // it there directly (no path reads y back when there is no residual; the
    // tensor-core path's combine stores 16-byte vectors, hence the alignment)
    void* ymap = nullptr;
    if ((reinterpret_cast<uintptr_t>(y_host) & 15) != 0 ||
        cudaHostGetDevicePointer(&ymap, y_host, 0) != cudaSuccess || !ymap) {
        (void)cudaGetLastError();
        ymap = nullptr;
    }
    if ((rc = coli_moe_forward_ex(layer, xd, xt, T, ymap ? static_cast<float*>(ymap) : yd, nullptr,
                                  path, nullptr, nullptr, nullptr, ws, inner, stream)))
        return rc;
    return ymap ? COLI_OK : stage_copy(yd, y_host, (size_t)row, false, S(stream));
}

int coli_moe_stack_host_workspace_size(const coli_moe_layer* const* layers, int32_t L, int32_t T,
                                       size_t* bytes) {
    size_t b;
    int rc = coli_moe_stack_workspace_size(layers, L, T, &b);
    if (rc) return rc;
    *bytes = (size_t)(align256((int64_t)b) + align256((int64_t)T * layers[0]->d.H * 4));
    return COLI_OK;
}

int coli_moe_stack_forward_host(const coli_moe_layer* const* layers, int32_t L,
                                const float* x_host, float* y_host, int32_t T, float eps,
                                coli_path path, void* ws, size_t ws_bytes, coli_stream_t stream) {
    if (!x_host || !y_host) return fail(COLI_E_INVAL, "stack_forward_host: NULL pointer");
    size_t need, inner;
    int rc = coli_moe_stack_host_workspace_size(layers, L, T, &need);
    if (rc) return rc;
    if ((rc = coli_moe_stack_workspace_size(layers, L, T, &inner))) return rc;
    if (!ws || ws_bytes < need)
        return fail(COLI_E_WORKSPACE, "stack_forward_host: workspace %zu < %zu bytes", ws_bytes, need);
    const size_t row = (size_t)T * layers[0]->d.H * 4;
    float* xd = reinterpret_cast<float*>(static_cast<char*>(ws) + align256((int64_t)inner));
    if ((rc = stage_copy(x_host, xd, row, true, S(stream)))) return rc;
    if ((rc = coli_moe_stack_forward(layers, L, xd, T, eps, path, ws, inner, stream))) return rc;
    return stage_copy(xd, y_host, row, false, S(stream));
}

int coli_moe_dequant_debug(const coli_moe_layer* layer, int32_t expert, int32_t which,
                           float* out, coli_stream_t stream) {
    if (!layer || !out) return fail(COLI_E_INVAL, "dequant_debug: NULL pointer");
    const coli_moe_desc& d = layer->run;
    const bool routed_here = expert >= layer->filter.e_lo && expert < layer->filter.e_hi;
    const bool shared_here = expert >= d.E && expert < d.E + d.n_shared;
    if (!(routed_here || shared_here) || which < 0 || which > 2)
        return fail(COLI_E_INVAL, "dequant_debug: expert %d / matrix %d out of range", expert, which);
    const BlobLayout& L = layer->L;
    const uint8_t* blob = layer->store.blob(expert);
    const int R = L.rows[which], K = L.cols[which];
    const int64_t n = (int64_t)R * K;
    auto kern = layer->bits == 8 ? dequant8_kernel : dequant_kernel;
    kern<<<(unsigned)((n + 255) / 256), 256, 0, S(stream)>>>(
        blob + L.codes[which], reinterpret_cast<const float*>(blob + L.scales[which]), R, K,
        d.group, out);
    return check_launch("dequant");
}

int coli_moe_union_readback(const coli_moe_layer* layer, int32_t T, const void* ws,
                            int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot,
                            int32_t* uniq, int32_t* n_uniq, int32_t* inv, coli_stream_t stream) {
    if (!layer || !ws) return fail(COLI_E_INVAL, "union_readback: NULL pointer");
    int rc = tokens_ok(layer->run, T);
    if (rc) return rc;
    const coli_moe_desc& d = layer->run;
    const WsPlan p = plan_ws(d, T);
    const char* w = static_cast<const char*>(ws);
    const int64_t Tk = (int64_t)T * d.k;
    struct { void* dst; int64_t off, n; } parts[] = {
        {offsets, p.offsets, d.E + 1}, {pair_tok, p.pair_tok, Tk}, {pair_slot, p.pair_slot, Tk},
        {uniq, p.uniq, d.E}, {n_uniq, p.n_uniq, 1}, {inv, p.inv, Tk}};
    for (auto& q : parts)
        if (q.dst && cudaMemcpyAsync(q.dst, w + q.off, (size_t)q.n * 4, cudaMemcpyDeviceToDevice,
                                     S(stream)) != cudaSuccess)
            return fail(COLI_E_CUDA, "union_readback: copy failed");
    return COLI_OK;
}

int coli_moe_status(const coli_moe_layer* layer, int32_t T, const void* ws, int32_t* flags,
                    coli_stream_t stream) {
    if (!layer || !flags) return fail(COLI_E_INVAL, "status: NULL pointer");
    int rc = tokens_ok(layer->run, T);
    if (rc) return rc;
    if (!ws) {  // the built-in scratch array of coli_moe_forward_noalloc
        void* scratch = nullptr;
        if ((rc = noalloc_scratch(&scratch))) return rc;
        ws = scratch;
    }
    const WsPlan p = plan_ws(layer->run, T);
    cudaStream_t st = S(stream);
    if (cudaMemcpyAsync(flags, static_cast<const char*>(ws) + p.err, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return fail(COLI_E_CUDA, "status: read failed");
    if (*flags & kErrWaitTimeout) return fail(COLI_E_TIMEOUT, "a device-side wait timed out; the outputs are invalid");
    return COLI_OK;
}


int coli_moe_forward_noalloc(const coli_moe_layer* layer, const void* x, coli_dtype xt,
                             int32_t T, float* y, coli_stream_t stream) {
    if (!layer || !x || !y) return fail(COLI_E_INVAL, "forward_noalloc: NULL pointer");
    int rc = tokens_ok(layer->run, T);
    if (rc) return rc;
    // the path AUTO would take if its workspace fits the array, else the
    // GEMV/GEMM path, whose workspace is a prefix of the full one
    coli_path path = COLI_PATH_AUTO;
    int64_t need = plan_ws(layer->run, T, kPlanFull).total;
    if (need > (int64_t)COLI_NOALLOC_SCRATCH_BYTES) {
        path = gemm_path_preferred(layer->run, T) ? COLI_PATH_GEMM : COLI_PATH_GEMV;
        need = plan_ws(layer->run, T, kPlanBase).total;
    }
    if (need > (int64_t)COLI_NOALLOC_SCRATCH_BYTES)
        return fail(COLI_E_UNSUPPORTED,
                    "forward_noalloc: T=%d needs %lld bytes of scratch, the built-in array holds %u",
                    T, (long long)need, (unsigned)COLI_NOALLOC_SCRATCH_BYTES);
    void* ws = nullptr;
    if ((rc = noalloc_scratch(&ws))) return rc;
    return coli_moe_forward_ex(layer, x, xt, T, y, nullptr, path, nullptr, nullptr, nullptr, ws,
                               (size_t)COLI_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
