/*
 * da2.h -- C ABI of the DraftAttention2 attention hot path for NVIDIA B200
 * (sm_100a).  Method: "DraftAttention2" (paperpeel.com/paper/2609.32628.md).
 *
 * The three calls follow the paper's statement of the problem (Sec. 3.1,
 * 3.3; App. C.1-C.2): per-head Q, K, V; a region partition of every frame;
 * operand preparation; draft-guided routing under precision budgets; one
 * block-sparse mixed-precision attention:
 *
 *   da2_prepare   -- fused gather + pooling + FP8/NVFP4 quantization (Sec. 3.3
 *                    "Fused quantization and reordering", Fig. 3b)
 *   da2_plan      -- draft map, per-head ranking, quotas, precision
 *                    assignment, per-row block lists (Eq. 3; Sec. 3.1 "Joint
 *                    allocation of sparsity and precision"; App. C.1)
 *   da2_attention -- phased FP8 / NVFP4 block-sparse attention with one
 *                    softmax state and one output accumulator, original token
 *                    order restored on store (Sec. 3.3 "Phased execution",
 *                    "Cross-precision accumulation"; App. B.3, C.1)
 *
 * Conventions for every call
 *   - Pointers marked (device) are CUDA device pointers, owned by the caller;
 *     the library never allocates on the call path.  The handle owns only
 *     its partition tables (allocated by da2_create, freed by da2_destroy).
 *   - All device work is asynchronous on the given stream; the call returns
 *     after enqueueing.  A stream of 0 means the legacy default stream.
 *     Calls on one handle must be ordered (same stream, or synchronized):
 *     the handle's small device work counter is shared by its launches.
 *   - Return value: DA2_OK or a negative DA2_ERR_* code; nothing is enqueued
 *     when an argument check fails.  DA2_ERR_CUDA means a launch failed; the
 *     CUDA error string is available from da2_last_cuda_error().
 *   - Device-side waits inside the kernels are bounded; when one gives up the
 *     kernel records it and returns; da2_check_device_status() reports it as
 *     DA2_ERR_TIMEOUT (it synchronizes the stream it is given).
 *   - Inputs are bf16, finite.  NaN / Inf inputs give undefined results.
 *
 * Geometry.  The sequence holds P prefix (text) tokens, then F frames of
 * Hv x Wv tokens in raster order (token t = P + f*Hv*Wv + y*Wv + x).  Each
 * frame is split into R_f = ceil(Hv*Wv/64) connected regions of balanced size
 * (App. C.2); region j of frame f is block a = f*R_f + j (Rv = F*R_f video
 * blocks); prefix block Rv + i holds prefix tokens 64i .. 64i+63; R = Rv +
 * ceil(P/64) blocks, Npad = 64*R packed slots.  Slots >= n_a of block a are
 * padding.
 */
#ifndef DA2_H
#define DA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DA2_OK 0
#define DA2_ERR_ARG -1     /* null pointer, bad shape, bad stride, budget > 100 %, C != 64, d not 64/128 */
#define DA2_ERR_ARCH -2    /* current device is not sm_100 */
#define DA2_ERR_CUDA -3    /* a CUDA call or launch failed */
#define DA2_ERR_TIMEOUT -4 /* a bounded device-side wait gave up */

typedef struct {
    int B, H;      /* batch, heads */
    int d;         /* head dim: 64 or 128 */
    int F, Hv, Wv; /* frames and latent frame size */
    int C;         /* region capacity = attention block size; must be 64 */
    int P;         /* prefix (text) tokens before the video tokens, 0 = none;
                      N = P + F*Hv*Wv tokens.  Pairs with a prefix block are not
                      counted in the precision budget (App. C.1): video queries keep every
                      prefix key and prefix queries attend to every key, on the
                      16-bit path (which then needs the bf16 operands). */
} da2_shape;

typedef struct {
    int bp_fp8;    /* basis points of the R^2 region pairs of each head kept in FP8 */
    int bp_fp4;    /* basis points kept in NVFP4; bp_fp16 + bp_fp8 + bp_fp4 <= 10000; the rest
                      is skipped */
    double lambda; /* max-pool branch weight of the draft map (Eq. 3); 0 = average only */
    int per_row;   /* 0: rank all R^2 pairs of a head together (DraftAttention2, Sec. 3.1
                      and App. C.1: one ranking per head).  1: rank the R key
                      blocks of each query block separately, quotas floor(R bp/10^4) per row
                      (a reading of a per-query-row ranking; ties to the smaller key block). */
    int bp_fp16;   /* basis points kept at 16 bits (bf16 operands; Table 1's 16-bit share),
                      the highest-ranked pairs; 0 = no 16-bit tier.  Cumulative cuts:
                      C16 = floor(n bp_fp16/10^4), C8 = floor(n (bp_fp16+bp_fp8)/10^4),
                      Ck = floor(n (bp_fp16+bp_fp8+bp_fp4)/10^4), n = R^2 (or R per row);
                      rank < C16 -> 16, < C8 -> 8, < Ck -> 4, else skipped (App. B.6). */
} da2_budget;

typedef struct da2_ctx* da2_handle;

/* Byte sizes of every caller-owned buffer for a shape (filled by da2_sizes).
 * R counts every block: the Rv video blocks, then the Rp = ceil(P/64) prefix
 * blocks; the draft map, the ranking and prec cover the Rv video blocks. */
typedef struct {
    int R, Rf, Npad;
    /* prepared operands */
    size_t desc, q8, k8, v8, q4, k4, v4, sfq, sfk, sfv, scale, vmax;
    /* plan outputs and scratch; kidx is the largest list size over all budgets
       (every pair kept): da2_list_bytes gives the exact size of a budget */
    size_t prec, cnt, off, kidx, A, plan_scratch;
    /* optional bf16 operands of the 16-bit path */
    size_t q16, k16, v16;
    /* optional INT8 operands of the 8-bit phase's QK^T */
    size_t q8i, k8i, si8;
    int Rv, Rp;
} da2_sizes_t;

/* Prepared operands (da2_prepare output, da2_attention input).  All device.
 *   desc  f64 [4][B][H][R][d]   Qbar, Qmax, Kbar, Kmax (Eq. 2): mean over the
 *                               n_a valid slots (fp64 sum in slot order, then
 *                               one fp64 divide) and channel-wise max.
 *   q8,k8 u8 [B][H][R][64*d]    e4m3 codes of the 64 x d tile, tcgen05 K-major
 *                               no-swizzle layout: byte (row r, col c) at
 *                               ((r/8)*(d/16) + c/16)*128 + (r%8)*16 + c%16.
 *   v8    u8 [B][H][R][d*64]    e4m3 codes of V^T (d rows x 64 slots), same
 *                               layout with 64 columns.
 *   q4,k4 u8 [B][H][R][64*d/2]  e2m1 codes, two per byte (even column in the low
 *                               nibble), same layout over d/2 byte columns.
 *   v4    u8 [B][H][R][d*32]    e2m1 codes of V^T, same layout, 32 byte columns.
 *   sfq   u8 [B][H][R][64][d/16] ue4m3 scale of each 16-channel group of Q.
 *   sfk   u8 [B][H][R][512]     ue4m3 scales of K (16-channel groups) in the
 *                               tensor-memory copy atom: byte 16*(n%32) +
 *                               4*(2*(c/64) + n/32) + (c%64)/16 for key slot n,
 *                               channel c (bytes not covered are zero).
 *   sfv   u8 [B][H][R][512]     ue4m3 scales of V^T (16-slot groups): byte
 *                               16*(c%32) + 4*(c/32) + j/16 for channel c, slot j.
 *   scale f32 [6][B][H][R]      FP8 tile scales of Q, K, V (amax/448), then
 *                               NVFP4 tile scales of Q, K, V (amax/2688).
 *   vmax  f32 [2][B][H]         per head max of the FP8 and of the NVFP4 V tile
 *                               scales (the phase units are vmax/448, vmax/2688).
 *   q16,k16 u8 [B][H][R][128*d] optional: bf16 tiles of Q and K for the 16-bit
 *                               path (the input values as they are), same layout
 *                               with 2d-byte rows; slots >= n_a are zero.
 *   v16   u8 [B][H][R][128*d]   optional: bf16 V^T (d rows x 64 slots, 128-byte
 *                               rows), same layout.
 *                               The three are all null (no 16-bit path) or all set.
 *   q8i,k8i s8 [B][H][R][64*d]  optional: INT8 codes of Q and K for the 8-bit
 *                               phase's QK^T (App. C.1: INT8 QK^T, FP8 PV), same
 *                               layout as q8; code = RNE(x * (127/amax)) of the
 *                               tile, clamped to +-127.
 *   si8   f32 [2][B][H][R]      optional: their tile scales amax/127 (Q, K).
 *                               The three are all null (FP8 QK^T) or all set;
 *                               when set, da2_attention takes the 8-bit phase's
 *                               scores from them.
 */
typedef struct {
    double* desc;
    uint8_t *q8, *k8, *v8, *q4, *k4, *v4, *sfq, *sfk, *sfv;
    float* scale;
    float* vmax;
    uint8_t *q16, *k16, *v16;
    int8_t *q8i, *k8i;
    float* si8;
} da2_prepared;

/* Plan (da2_plan output, da2_attention input).  All device.
 *   prec    u8  [B][H][Rv][Rv] precision of video pair (a,b): 16, 8, 4 or 0 (skip)
 *   cnt     i32 [3][B][H][R]  per query block: number of FP8, of NVFP4 and of
 *                             16-bit key blocks (prefix blocks count as 16-bit)
 *   off     i64 [B][H][R+1]   list offsets: query block a of head (b,h) owns
 *                             kidx[off[b][h][a] .. off[b][h][a+1]); head (b,h)
 *                             starts at (b*H + h) * K, K = the pairs a head keeps
 *                             (its budgeted video pairs, plus Rv*Rp + Rp*R with
 *                             a prefix)
 *   kidx    u16 [B*H*K]       compact lists: row a's 16-bit key blocks ascending
 *                             (for a video row: its 16-bit video blocks, then
 *                             every prefix block), then its FP8 ones, then its
 *                             NVFP4 ones (the phase order of the attention); a
 *                             prefix row lists every block
 *                             (da2_list_bytes bytes for the budget)
 *   A       f64 [B][H][Rv][Rv] the draft map (Eq. 3), left readable after the call
 *   scratch                   plan_scratch bytes of working memory
 */
typedef struct {
    uint8_t* prec;
    int32_t* cnt;
    int64_t* off;
    uint16_t* kidx;
    double* A;
    void* scratch;
} da2_plan_bufs;

/* Validate the shape, build the region partition on the host (App. C.2
 * reading: balanced R_f regions, boustrophedon band walk, smallest total
 * perimeter among connected candidates) and copy the slot tables to the
 * current device.  *out receives the handle.  The handle also holds a status
 * word and a work counter that its kernels share: order the calls made on one
 * handle (one stream, or synchronize between streams), or use one handle per
 * stream.  Errors: DA2_ERR_ARG, DA2_ERR_ARCH, DA2_ERR_CUDA. */
int da2_create(const da2_shape* shape, da2_handle* out);

/* Host-only: the partition of a shape without a device.  Fills
 * slot_token[64*R] (token of each packed slot, -1 = padding) and n_a[R]
 * (valid tokens per block), R = F*ceil(Hv*Wv/64), and returns R; returns
 * DA2_ERR_ARG for a non-positive size.  Either pointer may be NULL. */
int da2_partition(int F, int Hv, int Wv, int32_t* slot_token, int32_t* n_a);

/* Free the handle and its device tables.  NULL is accepted. */
int da2_destroy(da2_handle h);

/* Sizes of every caller-owned buffer for the handle's shape. */
int da2_sizes(da2_handle h, da2_sizes_t* out);

/* Exact byte size of the compact lists (da2_plan_bufs.kidx) under a budget:
 * 2 bytes per kept pair, B*H*K pairs with K = floor(Rv^2 bp/10^4) (per_row =
 * 0) or Rv*floor(Rv bp/10^4) (per_row = 1), bp = bp_fp16 + bp_fp8 + bp_fp4,
 * plus Rv*Rp + Rp*R prefix pairs.  Errors:
 * DA2_ERR_ARG for a null argument or a budget da2_plan would reject. */
int da2_list_bytes(da2_handle h, const da2_budget* budget, size_t* bytes);

/* Host copies of the partition tables: slot_token[Npad] (token of each packed
 * slot, -1 for padding) and n_a[R] (valid tokens per block).  Either may be
 * NULL. */
int da2_tables(da2_handle h, int32_t* slot_token, int32_t* n_a);

/* Fused operand preparation (Sec. 3.3, Fig. 3b).  q, k, v: bf16 (device),
 * element (b,h,t,c) at p[b*s[0] + h*s[1] + t*s[2] + c] with strides s[] in
 * elements (s[3] must be 1; the base and s[2] must keep rows 16-byte aligned).
 * Gathers every 64-slot block through the partition, writes the pooled
 * descriptors and the FP8 / NVFP4 operands and scales into *out. */
int da2_prepare(da2_handle h, const void* q, const void* k, const void* v, const int64_t strides[4],
                const da2_prepared* out, void* stream);

/* Draft-guided routing (Eq. 3; Sec. 3.1; App. C.1): A in fp64 with a fixed
 * operation order, per-head ranking of all R^2 pairs by A (ties to the
 * smaller pair index a*R+b), quotas T8 = floor(R^2 bp_fp8/10^4),
 * Tkeep = floor(R^2 (bp_fp8+bp_fp4)/10^4); ranks below T8 -> FP8, below
 * Tkeep -> NVFP4, the rest skipped; per-row lists.  With budget->per_row = 1
 * the ranking and the quotas floor(R bp/10^4) are per query block instead.
 * With bp_fp16 > 0 the three cuts of da2_budget give 16-bit, FP8 and NVFP4
 * pairs.  Errors: DA2_ERR_ARG for a budget outside [0, 10000], lambda
 * outside [0, 1] or per_row other than 0 / 1. */
int da2_plan(da2_handle h, const da2_prepared* prep, const da2_budget* budget, const da2_plan_bufs* plan,
             void* stream);

/* Size of the working memory da2_plan_static keeps inside the library:
 * 32 MiB of device memory on every GPU where the library is used, held until
 * the process exits. */
#define DA2_PLAN_STATIC_BYTES (32u << 20)

/* da2_plan for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is a service of the library.  Some callers must not call
 * cudaMalloc at the moment they route: code recording a CUDA graph by stream
 * capture (allocation is not allowed while a capture is open), hosts that own
 * all device memory through their own pools and forbid plugins to allocate,
 * and latency-critical paths where cudaMalloc's implicit synchronization
 * would stall other streams.  This entry point computes exactly what da2_plan
 * computes (same kernels, same results) but takes no scratch buffer: its
 * working memory is a fixed DA2_PLAN_STATIC_BYTES array inside the library.
 * The caller still passes the prepared operands and the five outputs (prec,
 * cnt, off, kidx, A, device, layouts as in da2_plan_bufs).
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress); make that first call before any stream
 *     capture begins.
 *   - Every call reuses the same array and clears what must start at zero;
 *     two calls that overlap on the same GPU (different streams, threads or
 *     handles) race on it: order them.
 *   - Returns DA2_ERR_ARG, without enqueueing anything, when the current
 *     device is not the handle's device, or when the shape needs
 *     more working memory than DA2_PLAN_STATIC_BYTES (da2_sizes' plan_scratch
 *     tells how much: about B*H*R*R*8 bytes plus 33 KB per head).  Other
 *     errors as da2_plan. */
int da2_plan_static(da2_handle h, const da2_prepared* prep, const da2_budget* budget, uint8_t* prec, int32_t* cnt,
                    int64_t* off, uint16_t* kidx, double* A, void* stream);

/* Block-sparse mixed-precision attention (Sec. 3.3; App. B.3, C.1).  out:
 * bf16 (device), [B][H][N][d] with strides out_strides[] in elements
 * (out_strides[3] == 1); every token row is written (rows with no retained
 * valid key get zeros).  The persistent CTAs take their work items from the
 * handle's work counter, which the call resets on `stream`: two attention
 * calls on one handle that overlap on different streams would share it and
 * leave rows unwritten, so order them (or use one handle per stream). */
int da2_attention(da2_handle h, const da2_prepared* prep, const da2_plan_bufs* plan, void* out,
                  const int64_t out_strides[4], void* stream);

/* Synchronize `stream` and report whether a bounded device wait gave up
 * since the last call (DA2_ERR_TIMEOUT), clearing the flag. */
int da2_check_device_status(da2_handle h, void* stream);

/* Limit of every bounded device-side wait in the kernels launched with this
 * handle, in nanoseconds; 0 restores the default (4 s).  A wait that reaches
 * the limit makes its kernel stop, drain its own asynchronous copies and
 * tensor-core work, free its tensor memory and return; the next
 * da2_check_device_status reports DA2_ERR_TIMEOUT.  The paper has no
 * counterpart: this is a service of the library. */
int da2_set_wait_limit(da2_handle h, uint64_t limit_ns);

/* Self-test of that failure path, with no fault and no hang: enqueues on
 * `stream` one small kernel whose first warp waits, with limit_ns, on a
 * device barrier that nothing arrives on, and whose second warp waits on the
 * same barrier with a 1000 times longer limit and must stop as soon as the
 * first gives up.  The kernel returns after about limit_ns; the next
 * da2_check_device_status then reports DA2_ERR_TIMEOUT.  limit_ns must be in
 * (0, 10^9], else DA2_ERR_ARG.  The paper has no counterpart. */
int da2_selftest_wait_timeout(da2_handle h, uint64_t limit_ns, void* stream);

/* Static description of a status code. */
const char* da2_status_string(int status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* da2_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DA2_H */
