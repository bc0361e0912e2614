/*
 * sva.h -- C ABI of the hybrid linear/softmax token mixer (sm_100a).
 *
 * The method is the token mixer of "SANA-Video 2.0: Hybrid Linear Attention
 * with Attention Residuals for Efficient Video Generation": three of every four
 * layers are gated linear attention with a fixed-size state, every fourth layer
 * is a gated softmax "anchor", and Block Attention Residuals (AttnRes) route the
 * summaries of completed 8-layer blocks into later linear layers through one
 * query projection shared across depth. Sources: lode.cx summary, section "How
 * It Works"; ai-papers.net summary, sections "ハイブリッド線形アテンション" and
 * "ブロックアテンション残差"; the SANA-Video 2.0 abstract on the
 * thelatestinai.com listing. The pages give the structure but no formula; the
 * formulas each entry point implements are stated beside it.
 *
 * Conventions shared by every entry point
 *  - Tensors are token-major and row-major: a [B, N, W] activation is B*N rows
 *    of `ld` elements each (ld >= W), batch b starting at row b*N. Head h of a
 *    D = H*d wide activation owns columns [h*d, (h+1)*d).
 *  - Weights use the [out, in] layout of a linear layer, so y = x W^T.
 *  - dtype SVA_BF16: operands are bf16, accumulation is fp32. dtype SVA_F32:
 *    everything is fp32 (plain CUDA-core kernels, no TF32).
 *  - Ownership: the caller owns every buffer and the stream. The library
 *    allocates no device memory, keeps no pointer after a call returns, and
 *    launches everything on the given stream without synchronising (except
 *    sva_check_device_status). Device pointers must be 16-byte aligned and every
 *    ld must be a multiple of 16 bytes.
 *  - Validation happens on the host before anything is launched; a failed
 *    check returns an error and launches nothing.
 *  - Workspaces: the first SVA_STATUS_BYTES of every workspace hold a device
 *    status word. Each call clears it on the stream before its kernels run;
 *    a kernel whose bounded wait on an mbarrier runs out writes
 *    SVA_ERR_DEVICE_TIMEOUT there and returns (no trap). Read it with
 *    sva_check_device_status.
 *  - Errors: SVA_ERR_INVALID_ARGUMENT (null pointer, bad size, stride or
 *    alignment), SVA_ERR_UNSUPPORTED (a valid shape the library has no kernel
 *    for, e.g. bf16 with d != 128), SVA_ERR_WORKSPACE (ws too small),
 *    SVA_ERR_CUDA (a launch or runtime call failed; see sva_last_cuda_error).
 */
#ifndef SVA_H_
#define SVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sva_stream_t; /* same handle as cudaStream_t; NULL = legacy stream */

typedef enum {
  SVA_OK = 0,
  SVA_ERR_INVALID_ARGUMENT = 1,
  SVA_ERR_UNSUPPORTED = 2,
  SVA_ERR_WORKSPACE = 3,
  SVA_ERR_CUDA = 4,
  SVA_ERR_DEVICE_TIMEOUT = 5
} sva_status_t;

typedef enum { SVA_F32 = 0, SVA_BF16 = 1 } sva_dtype_t;

#define SVA_STATUS_BYTES 256

/* sva_attn_args.flags: q and k already hold phi(Q) = ReLU(Q), phi(K) = ReLU(K)
 * (linear attention only; lets a producer that applied the feature map skip it). */
#define SVA_FLAG_QK_FEATURES 1u

/* Arguments of one attention-core call over all B*H (batch, head) pairs. */
typedef struct {
  int B, N, H, d;        /* batch, tokens, heads, head dim; D = H*d           */
  sva_dtype_t dtype;
  const void* q;    int64_t ldq;   /* [B, N, >=D] queries                      */
  const void* k;    int64_t ldk;   /* [B, N, >=D] keys                         */
  const void* v;    int64_t ldv;   /* [B, N, >=D] values                       */
  const void* gate; int64_t ldg;   /* [B, N, >=D] gate logits G                */
  const void* residual; int64_t ldr; /* nullable [B, N, >=D]: out = residual + Y */
  void* out;        int64_t ldo;   /* [B, N, >=D] output Y, may alias residual */
  float eps;        /* linear attention: normaliser epsilon (e.g. 1e-6)       */
  float scale;      /* softmax anchor: logit scale; 0 means 1/sqrt(d)         */
  unsigned flags;   /* SVA_FLAG_*                                             */
  const void* wgate; int64_t ldw;  /* linear attention, nullable [B, N, >=H]:
                                      write-gate logits, one per token and head,
                                      in dtype; row stride ldw >= H elements   */
  int n_keys;       /* softmax anchor: rows of k and v ([B, n_keys, >=D]) when
                       the queries are a shard of the sequence; 0 means N     */
} sva_attn_args;

/*
 * Gated linear attention (non-causal), the O(N) layers of the hybrid
 * [ai-papers.net summary, section "ハイブリッド線形アテンション": a fixed-size
 * state, cost linear in the number of tokens; lode.cx summary, "How It Works":
 * three of every four layers]. Per (batch, head), with phi = ReLU:
 *     S = sum_t phi(K_t)^T V_t  (d x d),   z = sum_t phi(K_t)  (d)
 *     Y_t = phi(Q_t) S / (phi(Q_t) . z + eps)  *  sigmoid(G_t)   (per channel)
 *     out_t = Y_t (+ residual_t)
 * Write-gated variant (wgate not NULL): the gate sets how much each token
 * writes into the state [ai-papers.net summary, same section]; token t's term
 * in both S and z is scaled by omega_t = sigmoid(wgate[b, t, h]):
 *     S = sum_t omega_t phi(K_t)^T V_t,   z = sum_t omega_t phi(K_t).
 * Supported: SVA_BF16 with d = 128 (tcgen05 kernels), SVA_F32 with d in
 * {64, 128}. Any N >= 1. The workspace holds per-chunk partial states (fp32)
 * and, for SVA_F32, the reduced state (the bf16 read-out sums the partials
 * itself); size it with sva_linear_attn_workspace_bytes.
 * The softmax anchor ignores wgate.
 */
size_t sva_linear_attn_workspace_bytes(int B, int N, int H, int d, sva_dtype_t dtype);
sva_status_t sva_linear_attn_fwd(const sva_attn_args* args, void* ws, size_t ws_bytes,
                                 sva_stream_t stream);

/*
 * The two halves of sva_linear_attn_fwd, for callers that shard the tokens
 * (e.g. across GPUs): the state is a sum over tokens, so the states of the
 * shards, summed (an all-reduce), are the state of the whole sequence, and
 * each shard's queries then read it out. The state is fp32, per (batch,
 * head) d*d + d values: S row-major (row = d_k, column = d_v), then z; size it
 * with sva_linear_attn_state_bytes (1.58 MB for B = 1, H = 24, d = 128); it
 * must be 16-byte aligned.
 *   sva_linear_attn_state_fwd:   uses k, v (and wgate) of args->N tokens and
 *                                writes the state; q, gate, out are ignored.
 *   sva_linear_attn_readout_fwd: uses q, gate, out (and residual) of args->N
 *                                query tokens and a given state; k, v ignored.
 * Workspace as for sva_linear_attn_fwd with the same B, N, H, d, dtype.
 */
size_t sva_linear_attn_state_bytes(int B, int H, int d);
sva_status_t sva_linear_attn_state_fwd(const sva_attn_args* args, float* state, void* ws,
                                       size_t ws_bytes, sva_stream_t stream);
sva_status_t sva_linear_attn_readout_fwd(const sva_attn_args* args, const float* state, void* ws,
                                         size_t ws_bytes, sva_stream_t stream);

/*
 * Allocation-free variant of sva_linear_attn_fwd (same arguments, same
 * results) for callers that cannot allocate device memory when they run the
 * mixer: engines that plan all device memory at start-up and allow no
 * allocation afterwards, plugins handed a stream but no allocator, programs
 * whose memory pool belongs to another framework. The method has no
 * counterpart; this is a library convenience. The scratch is a 16 MiB
 * file-scope device array held by every GPU that loads the library until
 * exit; calls needing more return SVA_ERR_WORKSPACE before launching
 * anything. The first call on a device looks up the array's address (make it
 * before any stream capture); the address is kept with the device's current
 * context, and the first call after a device reset (a new context) looks it
 * up again. All calls on a device share the array: calls that overlap on the
 * GPU race and must be serialised by the caller.
 * Device-side timeouts are not reported by this entry point.
 */
sva_status_t sva_linear_attn_fwd_noalloc(const sva_attn_args* args, sva_stream_t stream);

/*
 * Gated softmax anchor (non-causal), every fourth layer of the hybrid
 * [lode.cx summary, "How It Works": gated softmax keeps exact token relations;
 * SANA-Video 2.0 abstract: periodic gated-softmax anchors at a 3:1 ratio]:
 *     Y_t = sum_s softmax_s(scale * Q_t . K_s) V_s  *  sigmoid(G_t)
 * over the N query rows of q (gate, out, residual) and the n_keys rows of k
 * and v (n_keys = 0: the same N tokens; otherwise e.g. one shard's queries
 * against the all-gathered keys and values of the whole sequence).
 * No N x N matrix is stored. Supported: SVA_BF16 with d = 128 (tcgen05 flash
 * kernel), SVA_F32 with d in {64, 128}. Workspace: the status word, and for
 * SVA_BF16 the last wave's key-split parts (each part's unnormalised O, running
 * max and row sum, combined by a merge kernel); size it with
 * sva_softmax_anchor_workspace_bytes, which bounds it over every key count.
 */
size_t sva_softmax_anchor_workspace_bytes(int B, int N, int H, int d, sva_dtype_t dtype);
sva_status_t sva_softmax_anchor_fwd(const sva_attn_args* args, void* ws, size_t ws_bytes,
                                    sva_stream_t stream);

/*
 * Projections of a mixer layer: y = x W^T with x [M, K] (row stride ldx),
 * W [Nout, K] (contiguous, the [out, in] layout), y [M, Nout] (row stride ldy).
 * Used for the fused [Q | K | V | G] projection (Nout = 4D) and the output
 * projection. fp32 accumulation. `relu_cols`: columns [0, relu_cols) of y get
 * ReLU applied in the epilogue (0 = none); the stack uses it to hand phi(Q),
 * phi(K) to the linear layers. bf16: K and Nout multiples of 64; any M >= 1.
 */
size_t sva_projection_workspace_bytes(void);
sva_status_t sva_projection_fwd(const void* x, int64_t ldx, const void* w, int64_t M,
                                int64_t Nout, int64_t K, void* y, int64_t ldy, int relu_cols,
                                sva_dtype_t dtype, void* ws, size_t ws_bytes, sva_stream_t stream);

/*
 * Output projection fused with the residual update of the fp32 residual
 * stream: h += x W^T, and, when h_copy is not NULL, h_copy = dtype(h) (the next
 * layer's input). h is fp32 [M, Nout] with row stride ldh; h_copy has row
 * stride ldc.
 */
sva_status_t sva_projection_residual_fwd(const void* x, int64_t ldx, const void* w, int64_t M,
                                         int64_t Nout, int64_t K, float* h, int64_t ldh,
                                         void* h_copy, int64_t ldc, sva_dtype_t dtype, void* ws,
                                         size_t ws_bytes, sva_stream_t stream);

/*
 * AttnRes key of one completed block for the shared-query router
 * [ai-papers.net summary, section "ブロックアテンション残差": one query
 * projection shared across depth]. The router logit of block b is
 * (h W_r^T) . s_b = h . (s_b W_r), so each block needs one key tensor
 *     k_b = s_b W_r        s_b, k_b: [rows, D] contiguous; W_r: [D, D]
 * computed once when the block completes. The workspace holds W_r^T (bf16
 * path); size it with sva_attnres_keys_workspace_bytes.
 */
size_t sva_attnres_keys_workspace_bytes(int D, sva_dtype_t dtype);
sva_status_t sva_attnres_keys(const void* s_b, const void* w_r, void* k_b, int64_t rows, int D,
                              sva_dtype_t dtype, void* ws, size_t ws_bytes, sva_stream_t stream);

/*
 * AttnRes routing into a linear layer of a later block [ai-papers.net summary,
 * section "ブロックアテンション残差": summaries of completed blocks are routed
 * into later linear layers; lode.cx summary, "How It Works"]. Per token t:
 *     alpha_{t,b} = softmax_b( h_t . k_b[t] / sqrt(D) ),   b < n_blocks
 *     u_t = h_t + sum_b alpha_{t,b} s_b[t]
 * h: fp32 [rows, D] (the residual stream); keys[b], summaries[b], u: [rows, D]
 * in dtype, contiguous; alpha (nullable): fp32 [rows, n_blocks].
 * 1 <= n_blocks <= 8. No workspace.
 */
sva_status_t sva_attnres_route(const float* h, const void* const* keys,
                               const void* const* summaries, int n_blocks, void* u, float* alpha,
                               int64_t rows, int D, sva_dtype_t dtype, sva_stream_t stream);

/*
 * The hybrid stack: tokens in, mixed tokens out [SANA-Video 2.0 abstract;
 * lode.cx summary, "How It Works"]. h_0 = x; for l = 1..L (1-based):
 *   kind(l) = softmax anchor if all_softmax or l % softmax_period == 0, else linear
 *   block(l) = ceil(l / attnres_block); summary s_c = h_{c*attnres_block}
 *   u = route(h_{l-1}; s_1..s_{c-1}) for linear layers of block c >= 2
 *       (AttnRes on), else h_{l-1}
 *   [Q | K | V | G] = u W_qkvg[l]^T;  Y = gated core;  h_l = h_{l-1} + Y W_o[l]^T
 * y = dtype(h_L). The residual stream h is kept in fp32 in the workspace.
 * Write-gated linear layers: when w_wg is not NULL, linear layer l is the
 * write-gated variant with logits u W_wg[l]^T (W_wg[l]: [H, D] in dtype;
 * the entries of anchor layers are not read and may be NULL). The logits come
 * out of the same GEMM as [Q | K | V | G].
 * Optional traces (any may be NULL): trace_o[l] receives o_l = Y W_o^T as
 * fp32 [B*N, D]; trace_y[l] receives Y as dtype [B*N, D]; trace_alpha[l]
 * receives the router weights fp32 [B*N, c-1] of routed layers.
 * Optional profiling: when prof_events is not NULL it holds 2*prof_capacity
 * cudaEvent_t handles created by the caller; launch i of the call is bracketed
 * by events 2i and 2i+1 on `stream`, and prof_kind[i] (host array) receives
 * its SVA_KERNEL_* class. The number of launches is written to *prof_count.
 */
typedef enum {
  SVA_KERNEL_PROJ_QKVG = 0,
  SVA_KERNEL_PROJ_OUT = 1,
  SVA_KERNEL_LINEAR_STATE = 2,
  SVA_KERNEL_LINEAR_READOUT = 3,
  SVA_KERNEL_ANCHOR = 4,
  SVA_KERNEL_ROUTE = 5,
  SVA_KERNEL_KEYS = 6,
  SVA_KERNEL_OTHER = 7,
  SVA_KERNEL_LINEAR_REDUCE = 8
} sva_kernel_class_t;

typedef struct {
  int B, N, H, d, L;
  sva_dtype_t dtype;
  int softmax_period;          /* 4 in the method; 0 = no anchors                */
  int attnres_block;           /* 8 in the method; 0 = AttnRes off               */
  int all_softmax;             /* 1 = every layer an anchor (quadratic baseline) */
  const void* const* w_qkvg;   /* L pointers, each [4D, D] in dtype              */
  const void* const* w_o;      /* L pointers, each [D, D] in dtype               */
  const void* w_r;             /* [D, D] in dtype; may be NULL if nothing routes */
  float eps;                   /* linear-attention epsilon                       */
  void* const* trace_o;        /* optional, L pointers                           */
  void* const* trace_y;        /* optional, L pointers                           */
  void* const* trace_alpha;    /* optional, L pointers                           */
  void* const* prof_events;    /* optional, 2*prof_capacity cudaEvent_t          */
  int prof_capacity;
  int* prof_kind;              /* optional host array [prof_capacity]            */
  int* prof_count;             /* optional host int                              */
  const void* const* w_wg;     /* optional, L pointers, each [H, D] in dtype     */
  int* launch_count;           /* optional host int: kernels the call launched
                                  (counted with or without prof_events)         */
} sva_stack_desc;

size_t sva_hybrid_stack_workspace_bytes(const sva_stack_desc* desc);
sva_status_t sva_hybrid_stack_fwd(const sva_stack_desc* desc, const void* x, void* y, void* ws,
                                  size_t ws_bytes, sva_stream_t stream);

/*
 * The stack over n batches held in HOST memory (a library convenience for
 * streaming callers; the pages have no counterpart): batch i is x_host[i]
 * ([B, N, D] in dtype, contiguous) and its output goes to y_host[i]. The copy
 * in of batch i+1 and the copy out of batch i-1 overlap the stack pass of
 * batch i (two staging slots in `staging`, which the caller owns: size it with
 * sva_hybrid_stack_host_staging_bytes). Host buffers should be page-locked
 * for the copies to overlap; pageable memory works but serialises. The call
 * is asynchronous: it creates two copy streams and a few events and releases
 * them before returning (the runtime frees them once their work is done);
 * `stream` runs the stack passes, and once its work up to this call is
 * complete every y_host[i] holds its result. ws as for sva_hybrid_stack_fwd.
 */
size_t sva_hybrid_stack_host_staging_bytes(const sva_stack_desc* desc);
sva_status_t sva_hybrid_stack_fwd_host(const sva_stack_desc* desc, const void* const* x_host,
                                       void* const* y_host, int n, void* ws, size_t ws_bytes,
                                       void* staging, size_t staging_bytes, sva_stream_t stream);

/* Synchronises `stream`, then reads the status word of `ws` (SVA_OK or the
 * first device-side error, e.g. SVA_ERR_DEVICE_TIMEOUT). */
sva_status_t sva_check_device_status(const void* ws, sva_stream_t stream);

/* Launches one block that waits, with the library's bounded mbarrier wait and a
 * limit of `timeout_us` microseconds, on a barrier that nothing arrives at; the
 * wait runs out and the kernel records SVA_ERR_DEVICE_TIMEOUT in ws's status
 * word and returns. Exercises the device-timeout path without faulting. */
sva_status_t sva_selftest_bounded_wait(void* ws, size_t ws_bytes, unsigned timeout_us,
                                       sva_stream_t stream);

const char* sva_status_string(sva_status_t status);
const char* sva_last_cuda_error(void); /* text of the last CUDA error seen by this thread */
int sva_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SVA_H_ */
