/*
 * coli_moe.h - C ABI of libcolimoe: one routed Mixture-of-Experts FFN layer with
 * int4 expert weights (GLM-5.2 shape: hidden 6144, 256 routed experts + 1 shared,
 * intermediate 2048, top-8), computed by hand-written sm_100a CUDA kernels.
 *
 * The layer, per token x (sources are web pages, cited by title and section):
 *   1. Router   - z = W_r x (f32), s = sigmoid(z), sel = s + b; the k experts with
 *                 the largest sel (ties to the lower index); weights
 *                 w_j = s_j / sum(s) * routed_scale when norm_topk, else s_j * scale.
 *                 ["解密GLM-5.2-colibri-int4-with-int8-mtp" 模型架构深度解析;
 *                  "github一周涨11k⭐️！25GB 内存跑 744B GLM-5.2 模型！" 三.1, 四.3]
 *   2. Union    - the batch's (token, slot) pairs grouped by expert, so every
 *                 distinct expert is read once for all positions that chose it.
 *                 [same article, 三.4 "Batch-union MoE"; "colibrì 實戰指南" 二]
 *   3. Dequant  - w = float(q) * s, q a signed int4 nibble, s an f32 scale per row
 *                 or per 64 columns.  ["jlnsrk/GLM-5.2-colibri-int4 - Hugging Face"
 *                 container paragraph and conversion note; "colibrì 實戰指南" 三]
 *   4. SwiGLU   - h = silu(W_g x) * (W_u x), silu(a) = a / (1 + exp(-a)).
 *   5. Combine  - y = sum_j w_j * (W_d h)_j + sum over shared experts (weight 1).
 *                 ["解密GLM-5.2-colibri-int4-with-int8-mtp" 模型架构深度解析: 1 shared]
 *
 * Conventions
 *  - Every function returns an int: COLI_OK (0) or a negative coli_status.
 *    coli_moe_last_error() gives a thread-local message for the last failure.
 *  - The caller owns every buffer.  Pointers documented as "device" must be CUDA
 *    device memory of the current device; "host" means ordinary host memory.
 *    Apart from the small coli_moe_layer handle (host memory), the library
 *    allocates nothing: calls that need scratch space take a device workspace
 *    whose size coli_moe_workspace_size() reports.
 *  - Device calls are asynchronous on the given stream (NULL = legacy default
 *    stream) and never synchronise the host.  Launch errors are returned;
 *    errors raised while kernels run surface at the next synchronisation.
 *  - Calls that share a workspace must not overlap on the GPU.
 *
 * Matrix conventions: row-major [out, in]; gate and up are [I, H], down is [H, I].
 *
 * Container (host) layout of one quantised matrix [R, K] (coli_moe_quantize):
 *    codes  U8  [R, K/2]    column c in byte c/2, even c in the low nibble,
 *                           two's-complement signed nibble in [-8, 7]
 *                           (the quantiser only emits [-7, 7])
 *    scales F32 [R, K/G]    G = K (group 0, one scale per row) or 64
 *
 * Device layout of one expert ("blob", coli_moe_pack_expert): the container
 * re-tiled so that one 16-byte load of a lane is one lane's share of a 16x16
 * tensor-core operand tile; its dequantised values are identical.
 *    For each matrix m in (gate, up, down) with R rows and K columns:
 *      codes_m  [R/128][K/64][8][32][16 bytes]: unit (t, s, b, l) belongs to
 *               rows r0 = 128t + 16b + l/4 and r1 = r0 + 8, and holds four
 *               32-bit words j = 0..3 for columns c0 = 64s + 16j + 4(l%4) ..
 *               c0+3; in word j, byte i holds column c0 + i: row r0's signed
 *               nibble in bits 4-7, row r1's in bits 0-3, i.e. bits 4p..4p+3
 *               hold the nibble of
 *                 p: 0 (r1,c0)   1 (r0,c0)   2 (r1,c0+1) 3 (r0,c0+1)
 *                    4 (r1,c0+2) 5 (r0,c0+2) 6 (r1,c0+3) 7 (r0,c0+3)
 *      scales_m [R/128][K/G][128] f32          scale of row 128t + r, group g
 *    Order: codes_gate, codes_up, codes_down, scales_gate, scales_up,
 *    scales_down; each section starts on a 256-byte boundary and the blob size
 *    is a multiple of 256 bytes.  All experts of a layer sit back to back in one
 *    device buffer: routed experts 0 .. E-1, then the shared experts.
 *
 * Limits: H and I multiples of 128; group 0 or 64; 1 <= k <= 32; k <= E <= 1024;
 * n_shared <= 4; 1 <= T <= 8192 tokens per call and E * ceil(T/32) <= 24576.
 */
#ifndef COLI_MOE_H
#define COLI_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* coli_stream_t; /* same object as cudaStream_t */

typedef enum coli_status {
    COLI_OK = 0,
    COLI_E_INVAL = -1,       /* bad argument, shape or pointer               */
    COLI_E_CUDA = -2,        /* a CUDA runtime call or launch failed          */
    COLI_E_NOMEM = -3,       /* host allocation failed                        */
    COLI_E_UNSUPPORTED = -4, /* valid request this build does not implement   */
    COLI_E_WORKSPACE = -5,   /* workspace missing or smaller than required    */
    COLI_E_TIMEOUT = -6      /* a device-side bounded wait gave up            */
} coli_status;

typedef enum coli_dtype { COLI_F32 = 0, COLI_BF16 = 1 } coli_dtype;

typedef enum coli_path {
    COLI_PATH_AUTO = 0,  /* FUSED when it applies; else TWOPASS for 65 to 1024
                            tokens where it applies; else GEMV below 48
                            tokens, else GEMM                                  */
    COLI_PATH_GEMV = 1,  /* per-unit int4 GEMV kernels (mma.sync, fp16 hi/lo
                            activation digits, f32 accumulation)               */
    COLI_PATH_GEMM = 2,  /* tcgen05 grouped GEMM, fp16 operands, f32 accumulate */
    COLI_PATH_FUSED = 3, /* one persistent kernel for top-k, union and experts,
                            then a combine kernel (mma.sync s8, exact int32
                            sums per stage); T <= 64, T * (k + n_shared) <= 640,
                            E <= 256, k <= 32, n_shared <= 4, H a multiple
                            of 256, I <= 4096; the only path of 8-bit layers */
    COLI_PATH_TWOPASS = 4 /* large batches: router and union kernels, then a
                            gate/up pass writing h and a down pass writing
                            each pair's output (the fused kernel's mma.sync s8
                            stage on chunks of 16 of a unit's pairs), then the
                            combine; E <= 256, n_shared <= 4, H and I
                            multiples of 256; 4-bit layers                     */
} coli_path;

/* Thread-local description of the last error returned on this thread. */
const char* coli_moe_last_error(void);

/* ------------------------------------------------------------------------ */
/* Container                                                                 */
/* ------------------------------------------------------------------------ */

/* Quantise a host row-major f32 matrix [rows, cols] into the container layout
 * ("jlnsrk/GLM-5.2-colibri-int4 - Hugging Face": U8 packed nibbles + F32 scales;
 * conversion note: np.rint, i.e. round half to even).  Per row (group 0) or per
 * 64 columns: s = max|w| / 7 (f32 division); q = rint(w / s) clamped to [-7, 7]
 * (f32 division, half to even); s == 0 gives q = 0.
 * Host pointers: w [rows*cols], packed [rows*cols/2], scales [rows*cols/G].
 * Errors: COLI_E_INVAL for NULL pointers, rows < 0, odd cols, group not 0/64 or
 * cols not a multiple of 64 when grouped. */
int coli_moe_quantize(const float* w, int64_t rows, int64_t cols, int32_t group,
                      uint8_t* packed, float* scales);

/* Bytes of one expert blob in the device layout (see top of file). */
int coli_moe_expert_bytes(int32_t H, int32_t I, int32_t group, size_t* bytes);

/* Re-tile one expert's three container matrices (host memory, as written by
 * coli_moe_quantize) into one blob in the device layout (host memory, size
 * coli_moe_expert_bytes).  The blob keeps the three matrices adjacent, as the
 * engine stores an expert ("colibrì 實戰指南" 二: one read per expert).
 * Errors: COLI_E_INVAL for NULL pointers or unsupported shapes. */
int coli_moe_pack_expert(int32_t H, int32_t I, int32_t group,
                         const uint8_t* gate_codes, const float* gate_scales,
                         const uint8_t* up_codes, const float* up_scales,
                         const uint8_t* down_codes, const float* down_scales,
                         void* blob);

/* Device-side quantise + pack of one expert from f32 masters (device memory:
 * gate, up [I, H], down [H, I]) straight into a device blob; bit-identical to
 * coli_moe_quantize followed by coli_moe_pack_expert.  Asynchronous. */
int coli_moe_quantize_expert_device(int32_t H, int32_t I, int32_t group,
                                    const float* gate, const float* up,
                                    const float* down, void* blob,
                                    coli_stream_t stream);

/* 8-bit weights (the engine keeps its MTP head at 8 bits): the container's
 * rule with 127 in place of 7 - per row (group 0) or per 64 columns
 * s = max|w| / 127 (f32 division), q = rint(w / s) in [-127, 127] (f32
 * division, half to even), s == 0 gives q = 0.  Host pointers: w and codes
 * [rows*cols] (one signed byte per weight, row-major), scales [rows*cols/G].
 * Errors: COLI_E_INVAL as for coli_moe_quantize. */
int coli_moe_quantize8(const float* w, int64_t rows, int64_t cols, int32_t group,
                       int8_t* codes, float* scales);

/* Blob of one expert with 8-bit codes: codes_gate, codes_up, codes_down (each
 * R*K bytes), then the three scale sections as in the 4-bit blob, every
 * section on a 256-byte boundary.  Codes in 8-bit fragment tiles: blocks of 16
 * rows x 64 columns ordered [R/128][K/64][8][32 lanes]; lane l of block b in
 * row tile T and 64-column step s (g = l / 4, u = l % 4) holds 32 bytes: for
 * each 32-column half h, four words i = 0..3 - i = 0: row r0 = 128T + 16b + g,
 * columns 64s + 32h + 4u .. +3; i = 1: row r0 + 8, same columns; i = 2: row
 * r0, columns 64s + 32h + 16 + 4u .. +3; i = 3: row r0 + 8, those columns -
 * byte j of a word being its first column + j (the lane's mma.sync m16n8k32
 * s8 A registers).  coli_moe_pack_expert8
 * re-tiles host codes and scales (as written by coli_moe_quantize8) into a
 * host blob of coli_moe_expert_bytes8 bytes.  A layer created with bits = 8
 * reads such blobs on the fused path (the codes are the tensor-core operands
 * as they are: no decode). */
int coli_moe_expert_bytes8(int32_t H, int32_t I, int32_t group, size_t* bytes);
int coli_moe_pack_expert8(int32_t H, int32_t I, int32_t group,
                          const int8_t* gate_codes, const float* gate_scales,
                          const int8_t* up_codes, const float* up_scales,
                          const int8_t* down_codes, const float* down_scales,
                          void* blob);

/* Device-side 8-bit quantise + pack of one expert from f32 masters (as for
 * coli_moe_quantize_expert_device): bit-identical to coli_moe_quantize8
 * followed by coli_moe_pack_expert8.  Asynchronous. */
int coli_moe_quantize_expert8_device(int32_t H, int32_t I, int32_t group,
                                     const float* gate, const float* up,
                                     const float* down, void* blob,
                                     coli_stream_t stream);

/* coli_moe_quantize_expert_device for an expert given as FP8 E4M3 codes with
 * one f32 scale per 128 x 128 block (the format of the checkpoint the int4
 * container is converted from): every weight becomes
 * w = e4m3(code) * bs[r / 128][c / 128] in f32 (the E4M3 value is exact; one
 * f32 multiply), then the container's rule applies (s = max|w| / 7 per row or
 * per 64 columns, q = rint(w / s)).  Device memory: gate, up [I, H] and down
 * [H, I] as row-major bytes; gate_bs, up_bs [ceil(I/128), ceil(H/128)] and
 * down_bs [ceil(H/128), ceil(I/128)] row-major f32.  Bit-identical to decoding
 * on the host and using coli_moe_quantize + coli_moe_pack_expert.  The NaN
 * codes (S.1111.111) give undefined blobs.  Asynchronous. */
int coli_moe_quantize_expert_fp8_device(int32_t H, int32_t I, int32_t group,
                                        const uint8_t* gate, const uint8_t* up,
                                        const uint8_t* down, const float* gate_bs,
                                        const float* up_bs, const float* down_bs,
                                        void* blob, coli_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Layer                                                                     */
/* ------------------------------------------------------------------------ */

typedef struct coli_moe_desc {
    int32_t H;             /* hidden size                                    */
    int32_t I;             /* expert intermediate size (routed and shared)   */
    int32_t E;             /* routed experts                                 */
    int32_t k;             /* experts per token                              */
    int32_t n_shared;      /* shared experts, always applied with weight 1   */
    int32_t group;         /* 0 = per-row scales, 64 = per-64-column scales  */
    float routed_scale;    /* multiplies the routed weights (1.0 for GLM-5.2)*/
    int32_t norm_topk;     /* 1: renormalise the k scores to sum to 1        */
    const float* router_w; /* device f32 [E, H]                              */
    const float* router_b; /* device f32 [E], selection bias                 */
    const void* experts;   /* device, (E + n_shared) blobs back to back      */
    int32_t bits;          /* bits per weight code: 0 or 4 (int4 blobs of
                              coli_moe_pack_expert), 8 (8-bit blobs of
                              coli_moe_pack_expert8; fused path only)         */
} coli_moe_desc;

typedef struct coli_moe_layer coli_moe_layer;

/* Validate a descriptor and make a handle (host memory only; the device
 * buffers it points to stay owned by the caller and must outlive it). */
int coli_moe_layer_create(const coli_moe_desc* desc, coli_moe_layer** out);
int coli_moe_layer_destroy(coli_moe_layer* layer);

/* Adaptive expert top-p for every later forward of this layer ("colibrì 實戰指南"
 * 三 and 五: `--topp 0.7`, 30-40% fewer expert bytes per token, lossy; the pages
 * name the option but give no rule).  Rule: of a token's k picks, keep the
 * shortest run of the largest renormalised weights w_j / sum(w) (equal weights:
 * the lower expert index first) whose total reaches p, at least one pick; the
 * kept picks keep their weights w_j, the others add nothing to y.  The totals
 * are formed in double, in that order, from the f32 weights, and compared with
 * (double)p.  0 < p <= 1 enables it; p = 0 (the default) disables it; other
 * values give COLI_E_INVAL.  Forward calls then report w_out = 0 for dropped
 * picks.  Host-only: changes the handle, not device memory. */
int coli_moe_layer_set_topp(coli_moe_layer* layer, float p);

/* Expert parallelism: restrict this handle to the routed experts
 * e_begin <= e < e_end (and to the shared experts when with_shared != 0).
 * experts (device) then holds only those blobs: e_end - e_begin routed blobs in
 * expert order, followed by the n_shared shared blobs when with_shared != 0.
 * Routing still covers all E experts (the router is replicated); a forward
 * computes y = sum of w_j o_j over the picks whose expert is in the range (and
 * the shared experts when with_shared, and the residual when given), so the
 * sum of the y of handles whose ranges partition [0, E), exactly one of them
 * with the shared experts and the residual, is the layer's output.  Forward
 * calls report w_out = 0 for picks outside the range.  Workspace sizes follow
 * the restriction (no shared pairs when with_shared == 0).  Host-only. */
int coli_moe_layer_set_partition(coli_moe_layer* layer, int32_t e_begin, int32_t e_end,
                                 int32_t with_shared, const void* experts);

/* Test of the device-side bounded waits (no counterpart on the source pages):
 * on later fused-path forwards of this layer, CTA 0's producer skips ring
 * stage withhold_stage (0 = its first; < 0 = none, the default), so nothing
 * ever completes that stage and the consumer warps' wait on it gives up; with
 * the option set, every wait of the fused kernel gives up after 4096 tries
 * instead of the default (about a second).  The call then returns normally,
 * its outputs are invalid and coli_moe_status reports COLI_E_TIMEOUT; the
 * next call without the option is unaffected.  4-bit layers only (a fused
 * forward of an 8-bit layer with the option set returns COLI_E_UNSUPPORTED).
 * Never needed in normal use.  Host-only. */
int coli_moe_layer_set_wait_test(coli_moe_layer* layer, int32_t withhold_stage);

/* Workspace bytes that coli_moe_route / coli_moe_forward need for T tokens
 * (enough for every path; the GEMV and GEMM paths use only a prefix, the
 * fused and two-pass paths that prefix and their own buffers after it). */
int coli_moe_workspace_size(const coli_moe_layer* layer, int32_t T, size_t* bytes);

/* Step 1 alone.  x device [T, H] (f32 or bf16); idx device i32 [T, k] ordered
 * by (sel desc, expert asc); w device f32 [T, k]. */
int coli_moe_route(const coli_moe_layer* layer, const void* x, coli_dtype xt,
                   int32_t T, int32_t* idx, float* w, void* ws, size_t ws_bytes,
                   coli_stream_t stream);

/* Step 2 alone, for idx device i32 [T, k] with entries in [0, E): offsets
 * [E+1] (exclusive prefix of per-expert counts), pair_tok / pair_slot [T*k]
 * (pairs sorted by expert, then token), uniq [E] (ascending experts with at
 * least one pair; entries past n_uniq are left untouched), n_uniq [1].  All
 * device i32.  Needs no workspace.  Out-of-range expert ids give undefined
 * (but in-bounds) output. */
int coli_moe_union(const int32_t* idx, int32_t T, int32_t k, int32_t E,
                   int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot,
                   int32_t* uniq, int32_t* n_uniq, coli_stream_t stream);

/* Steps 1-5: writes y device f32 [T, H] (overwrites; no accumulation).  A pick
 * whose weight is 0 (dropped by top-p, outside the handle's expert range, or a
 * zero routed weight) is not computed: it would add exactly nothing. */
int coli_moe_forward(const coli_moe_layer* layer, const void* x, coli_dtype xt,
                     int32_t T, float* y, void* ws, size_t ws_bytes,
                     coli_stream_t stream);

/* Stage boundaries of coli_moe_forward_ex, for optional event timing. */
typedef enum coli_stage {
    COLI_STAGE_ROUTER = 0,  /* router logits (+ the activation operand)   */
    COLI_STAGE_UNION = 1,   /* sigmoid/top-k, weights and batch union     */
    COLI_STAGE_GATEUP = 2,  /* gate/up expert kernel with SwiGLU          */
    COLI_STAGE_DOWN = 3,    /* down expert kernel (and the fused combine) */
    COLI_STAGE_COMBINE = 4, /* a separate combine, where the path has one */
    COLI_STAGES = 5
} coli_stage;

/* coli_moe_forward with options: path selects the expert kernels; residual
 * (device f32 [T, H] or NULL) is added to the output (it may alias y);
 * idx_out / w_out (device, may be NULL) receive the routing decision: the k
 * experts of every token and the weights as applied (0 for a pick not
 * computed by this call).
 * events (may be NULL) is an array of COLI_STAGES + 1 cudaEvent_t created by
 * the caller; events[s] is recorded on `stream` just before stage s and
 * events[COLI_STAGES] after the last one, so cudaEventElapsedTime(events[s],
 * events[s+1]) is the device time of stage s. */
int coli_moe_forward_ex(const coli_moe_layer* layer, const void* x,
                        coli_dtype xt, int32_t T, float* y,
                        const float* residual, coli_path path, int32_t* idx_out,
                        float* w_out, void* const* events, void* ws,
                        size_t ws_bytes, coli_stream_t stream);

/* RMSNorm with unit gain, per row: out = x / sqrt(mean(x^2) + eps).  Device f32
 * [T, H]; out may alias x. */
int coli_moe_rmsnorm(const float* x, int32_t T, int32_t H, float eps, float* out,
                     coli_stream_t stream);

/* L stacked layers on a residual stream x (device f32 [T, H], updated in
 * place): x <- x + layer_l(rmsnorm(x)) for l = 0 .. L-1.  All layers must share
 * H; ws must cover the largest coli_moe_workspace_size(layers[l], T) plus
 * 4*T*H bytes (reported by coli_moe_stack_workspace_size). */
int coli_moe_stack_workspace_size(const coli_moe_layer* const* layers, int32_t L,
                                  int32_t T, size_t* bytes);
int coli_moe_stack_forward(const coli_moe_layer* const* layers, int32_t L,
                           float* x, int32_t T, float eps, coli_path path,
                           void* ws, size_t ws_bytes, coli_stream_t stream);

/* coli_moe_forward_ex (no residual, no routing outputs) for x and y in host
 * memory: x_host [T, H] (f32 or bf16) is copied into staging at the end of the
 * workspace, the layer runs on the device, and y [T, H] f32 is copied back into
 * y_host, all asynchronously on `stream`; y_host holds the result once the
 * stream has reached the end of the call (synchronise it or wait on an event
 * recorded after it).  Page-locked host memory that is mapped into the
 * device's address space (cudaHostAlloc memory on a unified-address system,
 * or cudaHostRegister with cudaHostRegisterMapped) is read and written by a
 * small kernel through that mapping, which for the few kilobytes of a decode
 * step avoids the copy engine's start-up latency; other memory is copied with
 * cudaMemcpyAsync (pageable memory only outside stream capture).  Page-locked
 * buffers make the call capturable into a CUDA graph.  ws must cover
 * coli_moe_host_workspace_size(layer, T) bytes (the forward's workspace plus
 * the staging of x and y). */
int coli_moe_host_workspace_size(const coli_moe_layer* layer, int32_t T, size_t* bytes);
int coli_moe_forward_host(const coli_moe_layer* layer, const void* x_host, coli_dtype xt,
                          int32_t T, float* y_host, coli_path path, void* ws,
                          size_t ws_bytes, coli_stream_t stream);

/* coli_moe_stack_forward for a residual stream in host memory: x_host f32
 * [T, H] is copied into staging in the workspace, the L layers run on it in
 * place, and the result is copied to y_host (which may equal x_host), with the
 * same rules as coli_moe_forward_host.  ws must cover
 * coli_moe_stack_host_workspace_size(layers, L, T) bytes. */
int coli_moe_stack_host_workspace_size(const coli_moe_layer* const* layers, int32_t L,
                                       int32_t T, size_t* bytes);
int coli_moe_stack_forward_host(const coli_moe_layer* const* layers, int32_t L,
                                const float* x_host, float* y_host, int32_t T, float eps,
                                coli_path path, void* ws, size_t ws_bytes,
                                coli_stream_t stream);

/* Device-side status of the most recent coli_moe_forward* call that used this
 * workspace (ws planned for T tokens): copies the error flags to *flags (host)
 * after synchronising `stream`.  Returns COLI_E_TIMEOUT if a bounded wait inside
 * a kernel gave up (its outputs are then invalid), else COLI_OK.  ws == NULL
 * reads the flags of the built-in scratch array of coli_moe_forward_noalloc on
 * the current device (T as in that call). */
int coli_moe_status(const coli_moe_layer* layer, int32_t T, const void* ws,
                    int32_t* flags, coli_stream_t stream);

/* Test helper: the batch union a forward built, read back from its workspace
 * (ws planned for T tokens; device i32 outputs, each may be NULL): offsets
 * [E+1], pair_tok and pair_slot [T*k] (pairs of computed picks grouped by
 * expert, experts ascending, tokens ascending), uniq [E] (first n_uniq
 * entries), n_uniq [1] after a GEMV-, GEMM- or two-pass forward; inv [T*k] (the
 * pair of each pick, -1 for a pick not computed) after any path.  The fused
 * path keeps its union in shared memory, in the order the picks first name
 * their experts: only inv describes it.  Asynchronous. */
int coli_moe_union_readback(const coli_moe_layer* layer, int32_t T, const void* ws,
                            int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot,
                            int32_t* uniq, int32_t* n_uniq, int32_t* inv, coli_stream_t stream);

/* Test helper: dequantise matrix `which` (0 gate, 1 up, 2 down) of expert
 * `expert` (0 .. E + n_shared - 1) from the device blob into out (device f32,
 * row-major [R, K] in container order). */
int coli_moe_dequant_debug(const coli_moe_layer* layer, int32_t expert,
                           int32_t which, float* out, coli_stream_t stream);

/* coli_moe_forward for callers that cannot allocate device memory.  (The
 * method on the source pages has no counterpart to this call; it exists for
 * integration only.)  Some hosts cannot hand this library a workspace: a plugin
 * running inside a framework that owns every device allocation and exposes no
 * allocator, or a real-time serving loop that forbids allocator calls once it
 * has started.  This call allocates nothing: instead of a caller workspace it
 * uses a scratch array of COLI_NOALLOC_SCRATCH_BYTES (8 MiB) compiled into the
 * library, which every GPU that loads the library keeps until the process
 * exits.  x, y and the layer's buffers are still the caller's.
 *  - T is limited to what fits.  The call takes the path coli_moe_forward
 *    would take when coli_moe_workspace_size(layer, T) fits the array, else
 *    the GEMV or GEMM path, which needs only part of that workspace; when
 *    neither fits it returns COLI_E_UNSUPPORTED (GLM-5.2 shapes: T <= 22; the
 *    fused path for T <= 2).
 *  - The first call on each device looks up that device's copy of the array
 *    (cudaGetSymbolAddress with the device current); make that first call before
 *    any stream capture.  Later calls only launch kernels, until the device's
 *    context is created anew (after cudaDeviceReset), when the next call looks
 *    the array up again.
 *  - A bounded device-side wait that gave up is reported by
 *    coli_moe_status(layer, T, NULL, ...), which reads the array's flags.
 *  - All calls share the one array, and it keeps whatever the previous call left
 *    in it (every value a call needs cleared is cleared by its own kernels).
 *    Calls whose kernels overlap on the GPU (different streams, or different
 *    host threads on one device) race on the array: serialise them.
 * Results equal coli_moe_forward_ex with the path taken (see above). */
#define COLI_NOALLOC_SCRATCH_BYTES (8u << 20)
int coli_moe_forward_noalloc(const coli_moe_layer* layer, const void* x,
                             coli_dtype xt, int32_t T, float* y,
                             coli_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* COLI_MOE_H */
