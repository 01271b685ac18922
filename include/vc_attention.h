/*
 * vc_attention.h -- C ABI of the VC-Attention forward for NVIDIA B200 (sm_100a):
 * V-Smooth prep followed by an ExpCast-FP8 attention kernel.
 *
 * Method sources (prose only; no code or equations are published):
 *   chooseai.io news 7051 (VC-Attention), sections "核心方法之一：V-Smooth ..."
 *     and "核心方法之二：ExpCast-FP8 ..."
 *   theclarity.today, "Quantizing value residuals and casting softmax to FP8
 *     speeds Nunchux's attention kernel 1.46x on an H200"
 *   zerohour.day summary "Nunchux AI Introduces VC-Attention ...", key facts
 *   RuntimeWire, "Nunchux speeds video diffusion with value smoothing and FP8
 *     softmax casting", section "The arithmetic behind the speedup"
 *
 * The op is a drop-in, training-free replacement of a non-causal
 * self-attention call over one long token sequence; the clustering runs inside
 * the call (theclarity.today, V-Smooth paragraph).
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major, on the current CUDA device, and owned by
 *     the caller.  The library never allocates device or host memory; its only
 *     state is a cached driver entry point and the static scratch array of
 *     vc_attn_fwd_noalloc.
 *   - All GPU work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and runs asynchronously.  No entry point synchronises,
 *     except vc_check.
 *   - Pointers must be 16-byte aligned device pointers (256-byte aligned is
 *     recommended).  Inputs must be finite.
 *   - Return values: VC_OK, or an error code.  Argument errors are detected on
 *     the host before any launch.  Launch failures return VC_ERR_CUDA.
 *     A kernel whose internal wait exceeds params->wait_limit_ns records
 *     VC_ERR_DEVICE_TIMEOUT in the workspace status word, lets its own copies
 *     and tensor-core work land, frees its tensor memory and returns; its
 *     outputs are undefined.  While the status word holds an error, every
 *     later kernel that reads the workspace returns without work (its outputs
 *     stay as they were) until vc_check reports and clears the error.
 *
 * Shapes: B batches, H heads, N tokens, head dim d (64 or 128).  The hardware
 * block is `block` tokens (64 or 128) and equals the key/value tile of the
 * attention kernel.  T = ceil(N / block) blocks; Tp = T * block.
 */
#ifndef VC_ATTENTION_H
#define VC_ATTENTION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VC_ABI_VERSION 2

typedef enum {
    VC_OK = 0,
    VC_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, bad size or parameter */
    VC_ERR_UNSUPPORTED = 2,    /* d or block outside {64,128}, 4-bit residual with block != 128, not sm_100 */
    VC_ERR_CUDA = 3,           /* a CUDA runtime or driver call failed */
    VC_ERR_DEVICE_TIMEOUT = 4, /* a device-side wait ran out (see wait_limit_ns) */
    VC_ERR_WORKSPACE = 5       /* workspace smaller than vc_workspace_bytes() */
} vc_status;

/* Q, K, V and O layout: bf16 [B, H, N, d]. */
typedef struct {
    int32_t B, H, N, d;
} vc_shape;

typedef struct {
    int32_t C;             /* k-means clusters, 1 <= C <= min(N, 256) */
    int32_t iters;         /* k-means assignment passes, 1 <= iters <= 64 */
    int32_t block;         /* hardware block = KV tile: 64 or 128 tokens */
    int32_t beta;          /* ExpCast shift: byte = round(8z + 56 + beta); integer in [0, 70] */
    int32_t smooth;        /* 1 = V-Smooth; 0 = plain per-channel FP8 V (identity order, zero means);
                              2 = V-Smooth reusing the regroup already in the prep's perm (from an
                              earlier call on the same shape): no k-means, K/V quantised in that order */
    int32_t resid_fmt;     /* 0 = E4M3 residual; 1 = 4-bit NVFP4 residual (block 128 only) */
    int64_t wait_limit_ns; /* bound on any single device-side wait; 0 = 2 s; below 1000 ns no
                              wait at all: only a phase complete at its first poll passes */
} vc_params;

/*
 * V-Smooth prep outputs (device pointers, caller-owned).  Positions are in
 * regrouped order: position i holds original token perm[i].
 *   perm     int32 [B,H,N]        stable order by k-means cluster id
 *   labels   int32 [B,H,N]        cluster id of each original token (optional: may be NULL)
 *   k_fp8    uint8 [B,H,Tp,d]     E4M3 K rows in regrouped order; rows >= N are 0
 *   k_scale  fp32  [B,H,T]        per-block K scale: K ~= k_scale[b] * E4M3(k_fp8)
 *   vt_fp8   uint8 [B,H,d,Tp]     E4M3 V residual, channel-major (transposed);
 *                                 columns >= N are 0.  With resid_fmt 1:
 *                                 [B,H,d,Tp/2], E2M1 codes two a byte (token
 *                                 2i in the low nibble)
 *   v_mean   fp32  [B,H,T,d]      block means of V (kept in fp32)
 *   v_scale  fp32  [B,H,d]        per-channel residual scale:
 *                                 V[perm[i]] ~= v_mean[i / block] + v_scale * E4M3(vt_fp8[:, i])
 *   v_bscale uint8 [B,H,T,d,block/16]  resid_fmt 1 only (NULL otherwise): the
 *                                 UE4M3 scale of each 16-token run of a channel:
 *                                 V[perm[i]][c] ~= v_mean[i / block][c] + v_scale[c] *
 *                                   E4M3(v_bscale[i / block][c][(i % block) / 16]) * E2M1(code)
 *   (4-bit residual: the zerohour.day summary lists NVFP4 beside E4M3 for
 *   the per-channel residual; E2M1 and UE4M3 as in the OCP MX formats.)
 */
typedef struct {
    int32_t* perm;
    int32_t* labels;
    uint8_t* k_fp8;
    float* k_scale;
    uint8_t* vt_fp8;
    float* v_mean;
    float* v_scale;
    uint8_t* v_bscale;
} vc_prep;

/* ABI version of the loaded library (VC_ABI_VERSION). */
int vc_abi_version(void);

/* Static, human-readable name of a vc_status value. */
const char* vc_status_string(int status);

/* Byte sizes of the eight vc_prep buffers, in struct order, for this shape and
 * params (v_bscale is 0 bytes unless resid_fmt is 1).  bytes must point to 8
 * size_t.  Host only; no CUDA call. */
vc_status vc_prep_buffer_bytes(const vc_shape* shape, const vc_params* params, size_t* bytes);

/* Workspace size needed by vc_smooth_prepare, vc_attn_fwd and vc_attention
 * (the largest of the three).  The workspace holds k-means state, quantised Q
 * and the device status word; it must be zero-filled once before its first
 * use (the status word must start at 0) and may be reused across calls on the
 * same stream.  Host only. */
vc_status vc_workspace_bytes(const vc_shape* shape, const vc_params* params, size_t* bytes);

/*
 * V-Smooth prep (chooseai.io news 7051, V-Smooth section; zerohour.day key
 * facts: per-channel E4M3 residual after block-mean subtraction).
 *   K, V    bf16 [B,H,N,d] device input
 *   out     prep buffers to fill (labels may be NULL)
 * Per (b, h): k-means over the N value vectors (strided init
 * c_k = V[floor(k N / C)], `iters` assignment passes, squared Euclidean
 * distance, ties to the lowest cluster, empty clusters keep their centroid);
 * stable regroup by cluster id; per block: K amax scale and E4M3 K, V mean,
 * V residual; per channel: residual amax scale and E4M3 residual.  smooth 2
 * skips the k-means and the regroup and keeps out->perm (and out->labels) as
 * they are: a later denoising step reuses an earlier step's clustering (the
 * pages run V-Smooth only in the first quarter of the steps on B200 and call
 * its cost a scheduling trade-off: chooseai.io news 7051, 意义与局限).  perm
 * entries outside [0, N) are read as token 0.  With
 * resid_fmt 1 the residual is 4-bit: per channel s_c = amax_c / (6 * 448), and
 * each 16-token run of a channel an NVFP4 block (UE4M3 scale E4M3(amax/6),
 * E2M1 codes of y * (1/scale) with y = r / s_c).
 */
vc_status vc_smooth_prepare(const void* K, const void* V, const vc_shape* shape, const vc_params* params,
                            const vc_prep* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * ExpCast-FP8 attention forward over prepped K/V (chooseai.io news 7051,
 * ExpCast-FP8 section; theclarity.today: block means are restored inside
 * the online softmax, so V is read once).
 *   Q     bf16 [B,H,N,d] device input, original token order
 *   prep  outputs of vc_smooth_prepare for the same shape and block
 *   O     bf16 [B,H,N,d] device output, original token order
 * Per query row: E4M3 Q with a per-token scale; FP8 QK^T on tensor cores;
 * per tile an integer row reference M (raised online); each score maps to the
 * E4M3 probability byte max(0, round(A*s + 56 + beta - 8M)) with one FMA;
 * FP8 PV; row sums of the tile restore the block means; O = (v_scale * O_res +
 * sum_b l_b mu_b) / l.  Non-causal; keys >= N are masked.  With resid_fmt 1
 * the PV product is 4-bit (tcgen05 kind::mxf4nvf4): each 16-key run of a row's
 * P is re-coded from the ExpCast byte's E4M3 value to NVFP4 (UE4M3 scale
 * E4M3(max/6), E2M1 codes of p * (1/scale)), against the 4-bit residual.
 */
vc_status vc_attn_fwd(const void* Q, const vc_prep* prep, const vc_shape* shape, const vc_params* params, void* O,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * vc_attn_fwd over a block-sparse subset of key tiles (chooseai.io news 7051,
 * 意义与局限: VC-Attention stacks with sparse attention).
 *   tile_mask  uint8 [B, H, Tq, T] device input, Tq = ceil(N / 128) query
 *              tiles of 128 rows, T = ceil(N / block) key tiles in regrouped
 *              order (the hardware blocks of vc_smooth_prepare); nonzero keeps
 *              key tile t for every row of query tile q.
 * A dropped tile takes no part in the row's max, ExpCast weights, row sums or
 * mean restore; a row whose tiles are all dropped outputs 0.  All ones is
 * vc_attn_fwd.  resid_fmt 1 is not supported (VC_ERR_UNSUPPORTED).  The mask
 * must not change until the call has run.
 */
vc_status vc_attn_fwd_masked(const void* Q, const vc_prep* prep, const vc_shape* shape, const vc_params* params,
                             const uint8_t* tile_mask, void* O, void* workspace, size_t workspace_bytes,
                             void* stream);

/* vc_smooth_prepare followed by vc_attn_fwd on the same stream: the drop-in
 * attention call.  `scratch` receives the prep outputs. */
vc_status vc_attention(const void* Q, const void* K, const void* V, const vc_shape* shape, const vc_params* params,
                       const vc_prep* scratch, void* O, void* workspace, size_t workspace_bytes, void* stream);

/*
 * vc_attention from host memory, with the transfers overlapped with the
 * computation.  The pages describe no such entry point; it serves callers
 * whose tensors live in host memory (a per-call H2D of Q, K, V and a D2H of
 * O).  The B*H independent (b, h) problems are split into `groups`
 * consecutive runs.  Group g's Q, K, V are copied on `h2d_stream`, its V-Smooth
 * prep and attention run on `compute_stream` once they have landed, and its
 * O is copied back on `d2h_stream`.  So the copies of group g+1 and g-1
 * overlap the computation of group g.
 *   Qh, Kh, Vh   bf16 [B,H,N,d] host input; page-locked (pinned) memory, or
 *                the copies do not overlap
 *   Oh           bf16 [B,H,N,d] host output, written asynchronously
 *   Qd, Kd, Vd, Od, scratch, workspace   device buffers as for vc_attention
 *                (full shape); workspace >= vc_workspace_bytes(shape)
 *   groups       1 .. B*H (clamped); 1 = no overlap
 * Results equal those of vc_attention on the same inputs.  The call only
 * enqueues: Oh is complete when d2h_stream has reached the end of the call;
 * vc_check(workspace, d2h_stream) synchronises and reports device errors.
 * The dependencies between the three streams use CUDA events that the call
 * creates and releases (released events stay valid until they complete); it
 * allocates no memory.
 */
vc_status vc_attention_host(const void* Qh, const void* Kh, const void* Vh, void* Oh, const vc_shape* shape,
                            const vc_params* params, int groups, void* Qd, void* Kd, void* Vd, void* Od,
                            const vc_prep* scratch, void* workspace, size_t workspace_bytes, void* h2d_stream,
                            void* compute_stream, void* d2h_stream);

/*
 * Allocation-free variant of vc_attn_fwd, for callers that cannot allocate
 * device memory at call time: a host runtime that hands the op only its
 * input and output buffers and owns every other byte, or a real-time loop that
 * cannot afford cudaMalloc's implicit device synchronisation or its failure
 * under memory pressure.  The pages describe no such entry point; it is a
 * property of this library, not of the method.
 *
 * Arguments and results are those of vc_attn_fwd without the workspace: the
 * quantised Q, its scales and the status word live in a scratch array that
 * the library reserves statically, VC_NOALLOC_SCRATCH_BYTES per device, held
 * by every GPU that loads the library until the process exits.  The problem
 * must fit: 768 + B*H*N*(d + 4) bytes (rounded up) <= VC_NOALLOC_SCRATCH_BYTES,
 * else VC_ERR_WORKSPACE is returned before anything is launched.
 *
 * The first call on a device looks up the scratch address on that device
 * (make that first call before any stream capture).  Every call shares the
 * one array and clears its status word first, so calls that overlap on the
 * GPU (other streams, or other host threads) race and must be serialised by
 * the caller.  A device-side wait timeout is not reported by this entry
 * point; O is then undefined.  No cudaMalloc, cudaFree or allocating library
 * routine is called.
 */
#define VC_NOALLOC_SCRATCH_BYTES (16u << 20)
vc_status vc_attn_fwd_noalloc(const void* Q, const vc_prep* prep, const vc_shape* shape, const vc_params* params,
                              void* O, void* stream);

/* Synchronises `stream`, reads and clears the workspace status word, and
 * returns VC_OK or the recorded device error (VC_ERR_DEVICE_TIMEOUT). */
vc_status vc_check(void* workspace, void* stream);

/* Element-wise E4M3 encode of fp32 values (round to nearest even, saturate to
 * +-448), the encoder every quantiser above uses.  x fp32 [n] -> out uint8 [n]. */
vc_status vc_e4m3_encode(const float* x, uint8_t* out, int64_t n, void* stream);

/* Per-token E4M3 quantisation of Q, the first step of vc_attn_fwd (both
 * operands of QK^T in FP8: chooseai.io news 7051, ExpCast-FP8 section).  For
 * each token: amax over its d channels, q_fp8 = E4M3(q * (448 / amax)),
 * sq = amax / 448 (0 and all-zero codes for an all-zero row).
 *   Q      device, bf16 [tokens, d] row-major, 16-byte aligned
 *   q_fp8  device, uint8 [tokens, d] out, 16-byte aligned
 *   sq     device, fp32 [tokens] out, 4-byte aligned
 *   d      64 or 128
 * Asynchronous on `stream`.  VC_ERR_INVALID_ARG for null or misaligned
 * pointers or tokens < 0, VC_ERR_UNSUPPORTED for another d. */
vc_status vc_quantize_q(const void* Q, uint8_t* q_fp8, float* sq, int64_t tokens, int d, void* stream);

/* Element-wise ExpCast byte map used inside vc_attn_fwd:
 * out[i] = max(0, round_half_even(A[i] * s[i] + cb[i])), one fp32 FMA with the
 * rounding inside it.  cb must hold integers with |cb| < 2^22.
 * A, s, cb fp32 [n] -> out uint8 [n]. */
vc_status vc_expcast_bytes(const float* A, const float* s, const float* cb, uint8_t* out, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VC_ATTENTION_H */
