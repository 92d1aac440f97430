// Internal interface of the non-tensor-core kernels (aux_kernels.cu).
#pragma once

#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"

namespace ipttt {
namespace aux {

cudaError_t build_meta(uint8_t* flags, ChunkMeta* meta, const Shape& s, const int32_t* doc_starts, int n_doc,
                       const int32_t* row_cont, int* status, cudaStream_t st);
cudaError_t conv_target(int dtype, const void* X0, const void* cw, const uint8_t* flags, void* U, const Shape& s,
                        cudaStream_t st);
cudaError_t alpha_from_partials(const float* partials, float* alpha, int n, int npairs, float eta, float tau,
                                cudaStream_t st);
cudaError_t state_export(bool blocked, const float* S, float* out, const Shape& s, cudaStream_t st);
// A row-major fp32 [B][d][F] state into the update kernel's blocked layout (null: zeros).
cudaError_t state_import_blocked(const float* in, float* Sb, const Shape& s, cudaStream_t st);
cudaError_t state_snapshot(const float* Sb, void* snap_bf16, const Shape& s, cudaStream_t st);
// One chunk of the accumulated-state clip on the bf16 path (row-major fp32 state,
// B x d F): S = c (keep S + eta raw), c = tau / ||keep S + eta raw||_F when that
// exceeds tau (into alpha[b][chunk]); snap_bf16 (or null) receives bf16(S).  part
// holds B x 592 partial sums.
cudaError_t state_clip_step(float* S, const float* raw, double* part, float* alpha, const ChunkMeta* meta,
                            const Shape& s, int chunk, float eta, float tau, void* snap_bf16, cudaStream_t st);

// SM_ACC: out += sum; SM_ACC_L: the same on the rows of each chunk's last document segment.
enum SimtMode { SM_Z = 0, SM_V = 1, SM_RAW = 2, SM_APPLY = 3, SM_ACC = 4, SM_ACC_L = 5 };

// Strided fp32 GEMM for the all-fp32 path: out(m,n) = epilogue(sum_k A(m,k) B0(n,k),
// sum_k A(m,k) B1(n,k)), one batch row b per blockIdx.z.
struct SimtArgs {
  int M, N, K;
  const float* A;
  long long sam, sak, sab;
  const float* B0;
  long long s0n, s0k, s0b;
  const float* B1;  // may be null
  long long s1n, s1k, s1b;
  int mode;
  float* out;
  long long som, son, sob;
  float* out2;      // SM_APPLY: optional D
  const float* resid;  // SM_APPLY: optional residual added to out (same strides as out)
  const ChunkMeta* meta;
  int k, C, chunk;
  int row0;         // token index of m = 0 (SM_V, SM_APPLY)
};

cudaError_t simt_gemm(const SimtArgs& a, int batches, cudaStream_t st);
cudaError_t simt_update_state(float* S, const float* raw, double* part, float* alpha, const ChunkMeta* meta,
                              const Shape& s, int chunk, float eta, float tau, cudaStream_t st);
// The ablation that clips the accumulated state instead of each delta (IPTTT_FLAG_STATE_CLIP):
// S = c (keep S + eta raw), c = min(1, tau / ||keep S + eta raw||_F), c stored in alpha.
cudaError_t simt_update_state_clipped(float* S, const float* raw, double* part, float* alpha, const ChunkMeta* meta,
                                      const Shape& s, int chunk, float eta, float tau, cudaStream_t st);

}  // namespace aux
}  // namespace ipttt

namespace ipttt {
namespace aux {
cudaError_t mask_last_segment(int dtype, const void* in, void* out, const ChunkMeta* meta, const Shape& s,
                              cudaStream_t st);
cudaError_t stream_advance(long long* pos, int32_t* cont, int B, int T, cudaStream_t st);
// Context parallelism: S_in from the gathered shard aggregates (ranks
// [first_rank, rank) of each row), added to the snapshots of the chunks that
// continue the incoming document, and S_final (optional); plan is [4][B] int32.
cudaError_t cp_combine(const float* gathered, int world, int rank, const int32_t* plan, void* snap, int nslots,
                       float* Sfinal, const Shape& s, cudaStream_t st);
cudaError_t prescale_target(void* V, const float* alpha, const Shape& s, float eta, cudaStream_t st);
}  // namespace aux
namespace bwd {
// Backward of the layer (backward.cu): fp32 gradients of <gO, O> + <gS, S_final>.
size_t workspace_bytes(const Shape& s);
long long launches(const Shape& s, int dtype);  // kernels one call of run launches

// What the bf16 backward reads from the forward run into its workspace: Z, U, V
// (bf16, V zero outside each chunk's last segment), alpha [B][k], chunk metadata,
// start flags, and the bf16 state copies S_i in slot i of [nslots][B][d][F].
struct TcForward {
  const void *Z, *U, *V, *snap;
  const float* alpha;
  const ChunkMeta* meta;
  const uint8_t* flags;
  int nslots;
  bool deltas_ready;  // the forward's update wrote every chunk's V_L^T Z_L (bf16) into tc_delta_buffer
};
size_t tc_workspace_bytes(const Shape& s);
// Where run_tc keeps the per-chunk deltas V_L^T Z_L ([k][B][d][F] bf16) in its workspace.
void* tc_delta_buffer(uint8_t* ws, const Shape& s);
long long tc_launches(bool deltas_ready, bool has_gS);
cudaError_t run_tc(const Shape& s, float eta, float tau, const TcForward& f, const void* H, const void* X0,
                   const void* Wg, const void* Wu, const void* W0, const void* cw, const void* Wt, const void* gO,
                   const float* gS, float* gH, float* gX0, float* gWg, float* gWu, float* gW0, float* gcw,
                   float* gWt, uint8_t* ws, int* status, int num_sms, cudaStream_t st);
cudaError_t run(const Shape& s, int dtype, float eta, float tau, const void* H, const void* X0, const void* Wg,
                const void* Wu, const void* W0, const void* cw, const void* Wt, const int32_t* doc, int n_doc,
                const void* gO, const float* gS, float* gH, float* gX0, float* gWg, float* gWu, float* gW0,
                float* gcw, float* gWt, uint8_t* ws, int* status, cudaStream_t st);
}  // namespace bwd
namespace aux {
// Grouped scan (short chunks taken gs.C tokens at a time, gs.C <= 1024): metadata
// of the groups (gs: the shape with C = the group length) and, per token, the
// offset in its group of the first token of its document within the group.
cudaError_t group_meta(const uint8_t* flags, ChunkMeta* gmeta, uint16_t* glo, const Shape& gs, cudaStream_t st);
}  // namespace aux
}  // namespace ipttt
