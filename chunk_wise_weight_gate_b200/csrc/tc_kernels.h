// Internal interface between the C-ABI layer and the tensor-core kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace ipttt {
namespace tck {

// FAM_ZV2: the gate/up and target GEMMs of FAM_ZV on CTA pairs (256-row tiles,
// M=256 pair MMAs, 128 K per stage); launched as clusters of two.
// FAM_GRAM2: the Gram pass on 256 x 256 token-block pairs, one cluster of two per
// block pair; each CTA writes its own partial (2 per pair, npairs = pairs per chunk).
// FAM_PZ: per group of gl tokens of a row (gl a multiple of 256), the masked
// token-token products P[t][u] = z_t . z_u for u in t's document and in an
// earlier chunk of the group (cta pairs, K = d_ff, 256 x 256 blocks on and below
// the diagonal), written as bf16 [B][T][gl]; the grouped scan's within-group term.
enum Family { FAM_ZV = 0, FAM_GRAM = 1, FAM_APPLY = 2, FAM_APPLY256 = 5, FAM_ZV2 = 6, FAM_GRAM2 = 8, FAM_PZ = 9 };

struct TcParams {
  CUtensorMap map[8];     // map[6]: the apply's O as 32-row x 64-column store boxes (o_tma);
                          // map[7]: the update's raw deltas [k B][d][F] as the same boxes (delta_out)
  int kind;          // FAM_ZV: kind_gateup() or kind_vhat()
  int vn;            // FAM_ZV target GEMM: output columns per tile (128 or 256)
  int B, T, d, F, C, k;
  int tr;            // token rows per apply / Gram tile: 128, or 64 when C % 128 != 0
  int ct;            // tiles per chunk (C / tr)
  int npairs;        // GRAM: tile pairs per chunk, ct (ct + 1) / 2
  int chunk;         // update: first chunk whose state update the launch performs
  int dchunks;       // update: consecutive chunks per launch
  int apply_chunk0;  // apply: first chunk of the launch's tiles
  int n_tiles;
  int nslots;        // apply, update: snapshot ring slots; S_i lives in slot i % nslots
  float eta;
  const ChunkMeta* meta;  // [B][k]
  const float* alpha;     // [B][k]
  float* partials;        // GRAM output [B][k][npairs]
  void* out0;             // Z (gate/up), V (target), O (apply)
  float* out1;            // apply: optional fp32 D
  const void* resid;      // apply: optional residual H added to O
  float* S;               // update: fp32 state, blocked 128 x 128 tiles
  int* status;            // device status word
  const void* src0;       // fused target: X0 [B][T][d]
  const void* src1;       // fused target: conv_w [d][5]
  const uint8_t* flags;   // fused target: document-start flags [B][T]
  const uint16_t* glo;    // FAM_PZ: per token, its document's first token within its group (offset)
  int cs;                 // FAM_PZ: chunk length
  int gl;                 // FAM_PZ, K_INTRA: tokens per group of the grouped scan
  const void* intra;      // apply: optional within-group term E [B][T][d] bf16, added to the fast-weight part
  int upd_kb;             // update: tokens per stage (0: update_tokens_per_stage(C))
  int upd_scale;          // update: 1 = V is not pre-scaled; the delta is scaled by alpha[b][chunk] eta
  int o_tma;              // 256-row apply: O leaves through shared memory and TMA stores (map[6])
  int delta_out;          // update: each chunk's raw delta V_L^T Z_L also goes out, bf16 (map[7])
  int rev;                // update: the backward's reverse scan (map[3] = gO_F, S = the start state G_k;
                          // slot i of map[5] receives bf16(G_{i+1}))
};

bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                   uint32_t box_inner, uint32_t box_rows);
cudaError_t launch_tc(int fam, const TcParams& p, int num_sms, cudaStream_t st);
// Whether FAM_ZV2 can run on this device (a cluster of two fits), and the
// number of CTA pairs resident at once.
int pair_gemm_workers(cudaStream_t st);
// State update of chunks [p.chunk, p.chunk + p.dchunks) on p.n_tiles state tiles of
// 128 x 256 (V pre-scaled by alpha eta); writes S_{c+1} snapshots and the fp32 state.
cudaError_t launch_update(const TcParams& p, int num_sms, cudaStream_t st);
// Tokens per pipeline stage of the state update for chunk length C: the V and Z
// tensor maps (map[3], map[4]) carry boxes of that many rows.
int update_tokens_per_stage(int C);
// Target GEMM with the masked conv in its producer (tgt_kernel.cu): V = conv(X0)
// Wtarget, rows outside each chunk's last segment zeroed.  map[0]: Wtarget, box
// {64, 64}; src0 X0, src1 conv_w, flags, meta, out0 V; n_tiles = B ceil(T/256)
// ceil(d/512).  Needs clusters of two and d % 256 == 0.
bool fused_target_supported(int d);
int fused_target_workers(cudaStream_t st);
cudaError_t launch_fused_target(const TcParams& p, cudaStream_t st);
cudaError_t launch_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t st);
int kind_gateup();
int kind_vhat();
int kind_intra();

}  // namespace tck
}  // namespace ipttt
