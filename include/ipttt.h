/*
 * ipttt.h -- C ABI of libipttt.so, the B200 (sm_100a) forward of one In-Place
 * Test-Time-Training MLP layer: a gated MLP whose down projection is a fast
 * weight updated chunk by chunk.
 *
 * What one call computes, for every row b of a batch of B sequences of T tokens
 * (sources: lijianxiong.blog notes "In-Place Test-Time Training", section 方法:
 * gated MLP, step 1 "apply", step 2 "update", the LM-aligned target and the
 * Hebbian rule, and 工程实现 for the exclusive prefix sum; cloud.tencent.com
 * "榨干MLP的剩余价值", 详细步骤 3 (depthwise conv, kernel 5, no look past the chunk)
 * and 4 (Frobenius clip); iplexlaw.co.kr review of arXiv 2604.06169, section 3
 * (apply before update) and section 6 (exclusive scan, document reset, clip)):
 *
 *   Z   = SiLU(H Wgate^T) * (H Wup^T)                              [T, F]
 *   U[t,c] = sum_{o=0..4} conv_w[c,o] * X0[t+o,c]   (tap zero when t+o is past the
 *            chunk end, past T, or in another document)
 *   V   = U Wtarget                                                  [T, d]
 *   chunks i = 0..k-1 of C tokens (the last may be short), k = ceil(T/C);
 *   S_0 = 0;   O_[i] = Z_[i] Wdown0^T + M_i * (Z_[i] S_i^T)          (pre-update state)
 *   dW_i = eta V_L^T Z_L over the rows L of the chunk's last document segment,
 *          scaled by alpha_i = tau/||dW_i||_F when ||dW_i||_F > tau (clip on)
 *   S_{i+1} = (chunk i holds a document start ? 0 : S_i) + alpha_i dW_i
 * M_i selects the rows of chunk i that belong to a document begun before the
 * chunk; rows of a document begun inside the chunk use Wdown0 alone.  A row start
 * is always a document start.
 *
 * Conventions for every entry point:
 *  - Tensors are DEVICE pointers owned by the caller, row-major and contiguous,
 *    16-byte aligned.  H, X0, O: [B, T, d].  Wgate, Wup: [F, d].  Wdown0: [d, F].
 *    conv_w: [d, 5] (tap o multiplies X0[t+o]).  Wtarget: [d, d], used as U Wtarget.
 *    All float tensors share params->dtype; O has that dtype.
 *  - doc_starts: DEVICE int32 array of n_doc_starts strictly increasing global
 *    token offsets b*T + t (row starts are implicit and may be omitted).
 *    Entries out of range or out of order make the call fail on the device
 *    (status IPTTT_ERR_ARG, see ipttt_get_status) and leave O unspecified.
 *  - The library allocates nothing.  Scratch memory is the caller's workspace
 *    (size from ipttt_workspace_size), 256-byte aligned, not shared between
 *    calls that may run concurrently.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Argument errors are returned synchronously and launch nothing.
 *    Errors found on the device (invalid doc_starts, a bounded wait that gave up)
 *    are recorded in a per-device status word read by ipttt_get_status.
 *  - Results are deterministic run to run (no floating-point atomics).
 *  - dtype IPTTT_F32 runs an all-fp32 path (SIMT FMA) for any shape.  dtype
 *    IPTTT_BF16 runs the tensor-core path (tcgen05, fp32 accumulation, fp32 fast
 *    weight state) and needs d % 128 == 0, F % 128 == 0, C % 64 == 0; other shapes
 *    return IPTTT_ERR_UNSUPPORTED.  Where the device runs clusters of two CTAs, the
 *    gate/up and target GEMMs, the Gram pass (C % 256 == 0) and the state update
 *    (d % 256 == 0) run on CTA pairs; the environment variables IPTTT_GEMM_CTAS=1
 *    and IPTTT_UPDATE_CTAS=1 select the single-CTA kernels instead.
 */
#ifndef IPTTT_H_
#define IPTTT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define IPTTT_API __attribute__((visibility("default")))
#else
#define IPTTT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  IPTTT_OK = 0,
  IPTTT_ERR_ARG = 1,          /* null pointer, non-positive size, bad eta/clip, bad doc_starts */
  IPTTT_ERR_SHAPE = 2,        /* sizes inconsistent or too large for 32-bit indexing */
  IPTTT_ERR_ALIGN = 3,        /* a tensor pointer is not 16-byte aligned (workspace: 256) */
  IPTTT_ERR_DTYPE = 4,        /* unknown dtype */
  IPTTT_ERR_UNSUPPORTED = 5,  /* shape outside what the bf16 tensor-core path handles */
  IPTTT_ERR_CUDA = 6,         /* a CUDA runtime call or a launch failed */
  IPTTT_ERR_TIMEOUT = 7,      /* a device-side bounded wait gave up */
  IPTTT_ERR_WORKSPACE = 8     /* workspace pointer null or smaller than required */
} ipttt_status;

typedef enum { IPTTT_F32 = 0, IPTTT_BF16 = 1 } ipttt_dtype;

typedef struct {
  int32_t B;          /* sequences in the batch                                  */
  int32_t T;          /* tokens per sequence (for streaming: tokens in this piece) */
  int32_t d;          /* d_model                                                  */
  int32_t F;          /* d_ff                                                     */
  int32_t C;          /* chunk size                                               */
  int32_t dtype;      /* ipttt_dtype                                              */
  float eta;          /* fast-weight learning rate                                */
  float clip_thresh;  /* Frobenius-norm threshold tau; <= 0 or +inf: no clip      */
  int32_t flags;      /* IPTTT_FLAG_* bits, 0 for none                            */
} ipttt_params;

/* O receives H + (layer output) instead of the layer output: the residual of a
 * stack of TTT layers, H_{l+1} = H_l + O_l, added in fp32 before the one rounding
 * to dtype.  O must not alias H. */
#define IPTTT_FLAG_RESIDUAL 1

/* The ablation that clips the accumulated fast weight instead of each chunk's
 * delta (iplexlaw.co.kr review of arXiv 2604.06169, §6, leaves open which of the
 * two the clip acts on): S_{i+1} = c_i (keep_i S_i + eta V_L^T Z_L) with
 * c_i = tau / ||keep_i S_i + eta V_L^T Z_L||_F when that norm exceeds tau, else 1.
 * Both dtypes; the per-chunk factor returned in alpha_opt is c_i.  On the bf16 path
 * each chunk's V_L^T Z_L is a tensor-core GEMM with an fp32 result and the state
 * update, norm and scale run on the CUDA cores in fp32, chunk by chunk.  The
 * context-parallel, decoding and backward entry points do not take it, nor does
 * streaming on the bf16 path (IPTTT_ERR_UNSUPPORTED). */
#define IPTTT_FLAG_STATE_CLIP 2

/* Bytes of workspace that ipttt_forward / _ex / stream_forward need for *p.
 * Returns 0 when *p is invalid.  Pure host function. */
IPTTT_API size_t ipttt_workspace_size(const ipttt_params* p);

/* One layer forward.  O: [B, T, d] output (device, dtype).  See the top of this
 * file for the computation and the argument conventions. */
IPTTT_API ipttt_status ipttt_forward(const ipttt_params* p,
                           const void* H, const void* X0,
                           const void* Wgate, const void* Wup, const void* Wdown0,
                           const void* conv_w, const void* Wtarget,
                           const int32_t* doc_starts, int32_t n_doc_starts,
                           void* O, void* workspace, size_t workspace_bytes,
                           void* stream);

/* ipttt_forward plus optional fp32 views of the internals, each NULL to skip:
 *   D_opt       [B, T, d]  the fast-weight term M_i * (Z_[i] S_i^T) of O
 *   S_final_opt [B, d, F]  the fast-weight state after the last chunk
 *   alpha_opt   [B, k]     the clip factor of every chunk (1 when not clipped)
 *   Z_opt       [B, T, F]  the gated activation (dtype)
 *   V_opt       [B, T, d]  the target V restricted to each chunk's last document
 *                          segment (other rows 0) (dtype)
 * The computation of O is the same code path as ipttt_forward. */
IPTTT_API ipttt_status ipttt_forward_ex(const ipttt_params* p,
                              const void* H, const void* X0,
                              const void* Wgate, const void* Wup, const void* Wdown0,
                              const void* conv_w, const void* Wtarget,
                              const int32_t* doc_starts, int32_t n_doc_starts,
                              void* O, float* D_opt, float* S_final_opt, float* alpha_opt,
                              void* Z_opt, void* V_opt,
                              void* workspace, size_t workspace_bytes, void* stream);

/* The chunk scan alone, with Z [B, T, F] and V [B, T, d] given (dtype); rows of V
 * outside a chunk's last document segment are ignored.  Same outputs as
 * ipttt_forward_ex.  Used to test the scan on hand-built activations such as the
 * induction-head setting of the notes' 理论分析 section. */
IPTTT_API ipttt_status ipttt_core(const ipttt_params* p, const void* Z, const void* V,
                        const void* Wdown0, const int32_t* doc_starts, int32_t n_doc_starts,
                        void* O, float* D_opt, float* S_final_opt, float* alpha_opt,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Streaming.  A caller-owned state carries each row's fp32 fast weight and
 * position between calls, so a long sequence can be fed in pieces; the result
 * equals one call over the whole sequence.  params->T is the piece length and
 * must be a multiple of C except for the final piece of a sequence (the conv
 * look-ahead and the update both close at chunk ends).  The bf16 path scans
 * chunks of 64, 128 or 256 tokens in groups of 512 tokens, starting at each
 * call's first token; pieces whose lengths are multiples of the scan group (512
 * tokens then, else C) give one call's result bit for bit, other whole-chunk
 * pieces give it up to rounding (the state sums and snapshots are grouped
 * differently).
 * doc_starts are offsets
 * b*T + t within the piece; a piece start is a document start only when the row
 * has consumed nothing yet or when doc_starts lists it.
 * State layout (opaque, 256-byte aligned): fp32 S[B][d][F], then per-row int64
 * position and int32 flags.  ipttt_stream_reset zeroes it (stream-ordered). */
IPTTT_API size_t ipttt_stream_state_size(const ipttt_params* p);
IPTTT_API ipttt_status ipttt_stream_reset(const ipttt_params* p, void* state, void* stream);
IPTTT_API ipttt_status ipttt_stream_forward(const ipttt_params* p, void* state,
                                  const void* H, const void* X0,
                                  const void* Wgate, const void* Wup, const void* Wdown0,
                                  const void* conv_w, const void* Wtarget,
                                  const int32_t* doc_starts, int32_t n_doc_starts,
                                  void* O, void* workspace, size_t workspace_bytes,
                                  void* stream);
/* Copies the state's fp32 S [B, d, F] to S_out (device). */
IPTTT_API ipttt_status ipttt_stream_export(const ipttt_params* p, const void* state, float* S_out,
                                 void* stream);

/* Context parallelism: the batch's sequences split along T over `world` ranks
 * (one process per GPU), rank r holding tokens [r*T, (r+1)*T) of every row, with
 * params->T the shard length (a multiple of C when world > 1, so that no conv tap
 * and no chunk crosses a shard).  The chunk deltas are independent of the state, so
 * each shard computes its own; the fast weight a shard starts from is the
 * segmented exclusive sum of the earlier shards' aggregates, restarted at the last
 * shard that holds a document start (lijianxiong.blog notes "In-Place Test-Time
 * Training", 工程实现: deltas in parallel, then a prefix sum; iplexlaw.co.kr
 * review §6: exclusive scan with document resets).  One exchange:
 *   ipttt_cp_begin   the shard's Z, V, clip factors and state updates from a zero
 *                    state; leaves the shard's aggregate in agg [B, d, F] fp32 (an
 *                    opaque tile order, the same on every rank);
 *   (caller)         all-gather agg in rank order into gathered [world, B, d, F];
 *   ipttt_cp_finish  adds the incoming state to the state the shard's chunks of the
 *                    continuing document see, applies every chunk (O [B, T, d] =
 *                    this shard's rows of the full forward) and optionally writes
 *                    S_final [B, d, F] (row-major fp32): the state after the shard's
 *                    last chunk (on the last rank, after the whole sequence).
 * doc_starts_host: HOST int32, n_doc_starts strictly increasing offsets
 * b*(world*T) + t over the whole sequence (every rank passes the same list).  Both
 * calls of a rank take the same params, world, rank, doc starts and workspace
 * (ipttt_cp_workspace_size bytes, 256-byte aligned; its snapshot ring holds the
 * state of every chunk of the shard), which must not be touched in between.
 * bf16 only (IPTTT_ERR_UNSUPPORTED otherwise).  Bad doc starts, world or rank
 * return IPTTT_ERR_ARG before anything is launched.  The incoming state is added
 * to the bf16 copy of each continuing chunk's state, one extra rounding against a
 * single-device forward.  H is read by the finish only with IPTTT_FLAG_RESIDUAL. */
IPTTT_API size_t ipttt_cp_workspace_size(const ipttt_params* p);
/* The host side of the split, run by both calls (pure host function): this rank's
 * document starts as offsets b*T + t within the shard (local_starts, room for
 * n_doc_starts entries, or NULL to count only; their number in *n_local), and
 * plan [4, B]: row_cont (the shard's first token continues a document), first_rank
 * (the first rank of the row's segmented sum), prefix_chunks (the shard's chunks
 * that see the incoming state) and keep (the incoming state reaches S_final). */
IPTTT_API ipttt_status ipttt_cp_plan(const ipttt_params* p, int32_t world, int32_t rank,
                                     const int32_t* doc_starts_host, int32_t n_doc_starts,
                                     int32_t* local_starts, int32_t* n_local, int32_t* plan);
IPTTT_API ipttt_status ipttt_cp_begin(const ipttt_params* p, int32_t world, int32_t rank,
                                      const int32_t* doc_starts_host, int32_t n_doc_starts,
                                      const void* H, const void* X0, const void* Wgate, const void* Wup,
                                      const void* conv_w, const void* Wtarget, float* agg,
                                      void* workspace, size_t workspace_bytes, void* stream);
IPTTT_API ipttt_status ipttt_cp_finish(const ipttt_params* p, int32_t world, int32_t rank,
                                       const int32_t* doc_starts_host, int32_t n_doc_starts,
                                       const void* H, const void* Wdown0, const float* gathered,
                                       void* O, float* S_final_opt,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* Waits for `stream`, then returns and clears the per-device status word that
 * kernels set on device-side errors (IPTTT_OK if none). */
IPTTT_API ipttt_status ipttt_get_status(void* stream);

/* Static description of a status code. */
IPTTT_API const char* ipttt_strerror(ipttt_status s);

/* The CUDA error behind the last IPTTT_ERR_CUDA returned on the calling thread:
 * the failing step and the CUDA runtime's error name and text ("" if none).  The
 * string belongs to the library and stays valid until the thread's next call. */
IPTTT_API const char* ipttt_last_error_detail(void);

/* Diagnostics.  While profiling is on, every call records CUDA events on its own
 * stream around each phase: 0 metadata (and, without CTA pairs, the conv), 1 gate/up
 * GEMM, 2 target GEMM (with the conv in its producer on CTA pairs),
 * 3 Gram pass + clip factors, 4 apply launches of the chunk scan, 5 state-update
 * launches of the chunk scan.  ipttt_profile_read waits for the recorded events
 * and returns, per phase, the milliseconds and kernel launches accumulated since
 * the previous read (n_phases <= 6); it returns the number of phases written.
 * ipttt_kernel_launches counts every kernel this library has launched in the
 * process. */
IPTTT_API void ipttt_profile_enable(int on);
IPTTT_API int ipttt_profile_read(double* ms, uint64_t* launches, int n_phases);
IPTTT_API uint64_t ipttt_kernel_launches(void);

/* Forward without any allocation, for callers that cannot call cudaMalloc: code
 * whose device memory belongs to another allocator (a framework's caching
 * allocator, a serving runtime with a fixed memory budget) and may not grow it in
 * the middle of a run, or a latency-critical path that cannot accept the implicit
 * device synchronisation of cudaMalloc/cudaFree.  The paper has no counterpart;
 * this is a packaging variant of ipttt_forward.
 *
 * Same arguments and result as ipttt_forward, minus the workspace: the library
 * uses its own scratch, a static device array of IPTTT_NOALLOC_SCRATCH_BYTES that
 * every GPU loading the library holds until the process exits.  Shapes whose
 * ipttt_workspace_size exceeds that return IPTTT_ERR_SHAPE without launching.
 * The scratch address is looked up once per device, on that device's first call
 * (make that call before any stream capture); the call allocates nothing.  All
 * calls on a device share the one scratch array and it keeps the last call's
 * contents (every call initialises what it reads), so calls that may overlap on
 * the GPU (different streams without ordering, or different host threads) race
 * and must be serialised by the caller. */
#define IPTTT_NOALLOC_SCRATCH_BYTES (32u << 20)
IPTTT_API ipttt_status ipttt_forward_noalloc(const ipttt_params* p,
                                   const void* H, const void* X0,
                                   const void* Wgate, const void* Wup, const void* Wdown0,
                                   const void* conv_w, const void* Wtarget,
                                   const int32_t* doc_starts, int32_t n_doc_starts,
                                   void* O, void* stream);

/* Self-test of the device-side failure path: launches one block that waits, with
 * the same bounded wait the kernels use, on a barrier phase that nothing ever
 * completes.  After limit_ns nanoseconds (0: the kernels' own limit, 2 s) it gives
 * up and records IPTTT_ERR_TIMEOUT in the status word (read it with
 * ipttt_get_status); the context stays usable.  Meant for tests. */
IPTTT_API ipttt_status ipttt_selftest_wait_timeout(uint32_t limit_ns, void* stream);

/* Host-buffer forward.  Same result as ipttt_forward, but H, X0 and O are HOST
 * arrays [B, T, d] (page-locked memory lets the copies overlap the compute; with
 * pageable memory the result is the same, only slower) and doc_starts is a HOST
 * int32 array with the meaning given above.  The weights are device pointers.
 * The pages have no counterpart: this is the way to feed a sequence that sits in
 * host memory without waiting for the whole of it to be copied first.
 *
 * The sequence runs through ipttt_stream_reset / ipttt_stream_forward in pieces of
 * piece_tokens tokens of every row (a multiple of C; 0 picks about T/8 in whole
 * scan groups, so that the result is ipttt_forward's bit for bit, see streaming
 * above): while piece i computes on `stream`, piece i+1 is copied in and piece
 * i-1 copied out on two streams the call creates and releases.  device_buffer is
 * caller-owned device memory, 256-byte aligned, of ipttt_forward_host_size(p,
 * piece_tokens, n_doc_starts) bytes (two device copies of a piece of H, X0 and O,
 * the pieces' document starts, the streaming state and a workspace); the call
 * allocates no device memory.  Document starts are checked on the host (out of
 * range or out of order: IPTTT_ERR_ARG, nothing launched).  The call returns once
 * everything is queued; later work on `stream` sees O complete.  H, X0, O and
 * device_buffer must stay untouched until then; doc_starts may be released when
 * the call returns. */
IPTTT_API size_t ipttt_forward_host_size(const ipttt_params* p, int32_t piece_tokens, int32_t n_doc_starts);
IPTTT_API ipttt_status ipttt_forward_host(const ipttt_params* p, const void* H_host, const void* X0_host,
                                          const void* Wgate, const void* Wup, const void* Wdown0,
                                          const void* conv_w, const void* Wtarget,
                                          const int32_t* doc_starts_host, int32_t n_doc_starts,
                                          void* O_host, void* device_buffer, size_t device_bytes,
                                          int32_t piece_tokens, void* stream);

/* Token-by-token decoding (bf16, B <= 16 rows decoded together).  The pages leave
 * the decode stage unmeasured (iplexlaw.co.kr review of arXiv 2604.06169, §7.5 and
 * §8); what it must compute follows from the ordering (§3, §9.1): a token inside
 * chunk i is output with the state committed before the chunk, and a chunk's delta
 * is committed once the chunk is complete.  Per step, for every row b:
 *   z = SiLU(Wgate h_b) * (Wup h_b)  (rounded to bf16),
 *   o_b = Wdown0 z + m_b (S_i z)     (one fp32 sum, rounded to bf16),
 * m_b = 1 while the row's document began before the current chunk.  When C tokens
 * have been decoded, the chunk's H and X0 rows (kept in the state) go through
 * ipttt_stream_forward, which commits S_{i+1} exactly as a prefill would; the
 * outputs then equal ipttt_forward's up to the fp32 summation order.
 *
 * State: a device buffer of ipttt_decode_state_size(p) bytes (256-byte aligned:
 * streaming state, the chunk's H and X0 rows, a bf16 copy of the committed state,
 * a workspace) and a host buffer of ipttt_decode_host_size(p) bytes (positions and
 * the chunk's document starts); p->T is ignored.  ipttt_decode_reset starts every
 * row afresh.  ipttt_decode_step takes h, x0 and writes o, DEVICE [B, d] bf16;
 * starts_host (HOST int32 [B], or NULL) flags rows whose token begins a new
 * document.  The step that completes a chunk copies that chunk's document starts
 * from the host buffer (pageable), so it first waits for work queued on `stream`.
 * Other shapes or dtypes: IPTTT_ERR_UNSUPPORTED.  ipttt_decode_export copies the
 * committed fp32 state [B, d, F] to S_out (device). */
IPTTT_API size_t ipttt_decode_state_size(const ipttt_params* p);
IPTTT_API size_t ipttt_decode_host_size(const ipttt_params* p);
IPTTT_API ipttt_status ipttt_decode_reset(const ipttt_params* p, void* state, void* host_state, void* stream);
IPTTT_API ipttt_status ipttt_decode_step(const ipttt_params* p, void* state, void* host_state,
                                         const void* h, const void* x0, const int32_t* starts_host,
                                         const void* Wgate, const void* Wup, const void* Wdown0,
                                         const void* conv_w, const void* Wtarget, void* o, void* stream);
IPTTT_API ipttt_status ipttt_decode_export(const ipttt_params* p, const void* state, float* S_out,
                                           void* stream);

/* Library version, "major.minor.patch". */
IPTTT_API const char* ipttt_version(void);

/* Backward of the layer (ipttt_forward's inputs, params->flags must be 0).  Given
 * gO = dL/dO ([B][T][d], the layer's dtype) and optionally gS_final = dL/dS_final
 * (fp32 [B][d][F] row-major; NULL = 0), writes the fp32 gradients of
 * L = <gO, O> + <gS_final, S_final> with respect to H and X0 ([B][T][d]), Wgate and
 * Wup ([F][d]), Wdown0 ([d][F]), conv_w ([d][5]) and Wtarget ([d][d]), through the
 * gated MLP, the chunk scan with its document resets, the per-chunk clip (the
 * derivative of the branch the forward took; the clip has a kink at norm tau), and
 * the masked conv target.  The pages give no backward: the layer is trained in
 * place (cloud.tencent.com "榨干MLP的剩余价值", 验证模块一), and these are the chain
 * rule through the forward defined above.  dtype IPTTT_F32 runs every product in
 * fp32 on the CUDA cores (any shape).  dtype IPTTT_BF16 (the forward's tensor-core
 * shapes) runs the forward first, keeping every chunk's bf16 state copy, then
 * every product as a tcgen05 GEMM on bf16 operands with fp32 accumulators: the
 * forward's Z and V, each chunk's raw delta V_L^T Z_L and the bf16 copies of the
 * state gradients are operands, so the gradients carry bf16 operand rounding.
 * Deterministic either way.  All pointers are device memory owned by the caller,
 * 16-byte aligned; workspace (256-byte aligned) of ipttt_backward_workspace_size(p)
 * bytes (fp32: k + 4 fp32 states [B][d][F]; bf16: three bf16 states [B][d][F]
 * per chunk (the forward's state copies, the raw deltas, the state-gradient copies),
 * one fp32 state, and about 20 F bytes per token of activations and their
 * gradients).  Errors as for ipttt_forward. */
IPTTT_API size_t ipttt_backward_workspace_size(const ipttt_params* p);
IPTTT_API ipttt_status ipttt_backward(const ipttt_params* p, const void* H, const void* X0, const void* Wgate,
                                      const void* Wup, const void* Wdown0, const void* conv_w,
                                      const void* Wtarget, const int32_t* doc_starts, int32_t n_doc_starts,
                                      const void* gO, const float* gS_final_opt, float* gH, float* gX0,
                                      float* gWgate, float* gWup, float* gWdown0, float* gconv_w,
                                      float* gWtarget, void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* IPTTT_H_ */
