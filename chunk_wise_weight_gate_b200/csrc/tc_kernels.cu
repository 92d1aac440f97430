// Tensor-core (tcgen05) kernels of the bf16 path of the In-Place TTT MLP layer.
//
// One persistent, warp-specialised kernel template serves the GEMMs of the layer.
// Per CTA: warp 0 issues TMA loads into a ring of shared-memory stages, warp 1
// allocates TMEM and one thread of it issues tcgen05.mma into fp32 accumulators,
// and 8 epilogue warps drain finished accumulators with tcgen05.ld.  Tiles are
// handed out statically (tile = worker + j * workers, a worker being a CTA or a
// cluster of two) and every role decodes the same tile index into the same Job.
// The pair families run as clusters of two CTAs: the even CTA issues M=256
// tcgen05.mma.cta_group::2, each CTA loads its 128 A rows and half of the N
// operand into its own shared memory (completion counted on the even CTA's
// barrier), MMA completions are multicast to both CTAs' barriers, and both CTAs'
// epilogues release the accumulator on the even CTA's barrier.
//
// Families (template parameter FAM):
//   FAM_ZV / FAM_ZV2 (pairs)  gate/up GEMM with the SiLU-product epilogue,
//            Z = SiLU(H Wg^T) * (H Wu^T) [notes "In-Place Test-Time Training",
//            方法 › 原地自适应], and the target GEMM V = U Wtarget with rows outside
//            each chunk's last document segment zeroed [notes, 对齐语言模型的目标函数].
//   FAM_GRAM / FAM_GRAM2 (pairs)  per-chunk Gram pass:
//            ||V_L^T Z_L||_F^2 = sum_{s,t}(V V^T)_{st}(Z Z^T)_{st}, written as
//            deterministic partial sums per tile pair; the clip factor follows
//            [cloud.tencent.com "榨干MLP的剩余价值", 详细步骤 4].
//   FAM_APPLY / FAM_APPLY256  apply tiles of a group of chunks:
//            O_i = Z_i W0^T + M_i (Z_i S_i^T), both products side by side in one
//            N=256 accumulator, S_i read from a bf16 snapshot [notes, 步骤一 and
//            工程实现; iplexlaw.co.kr review §3: a chunk's output comes from the
//            pre-update state].
// The state update S_{i+1} = keep_i S_i + alpha_i eta V_i^T Z_i runs in its own
// kernel (upd_kernel, below): the MMAs form each chunk's delta from zero in TMEM,
// and the epilogue warps hold the fp32 state of one tile in registers and add the
// deltas to it, walking the tile through a group of chunks [notes, 步骤二 and the
// Hebbian rule; iplexlaw.co.kr review §6 exclusive scan and document reset].
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "tc.cuh"
#include "tc_kernels.h"

namespace ipttt {
namespace tck {

using namespace ipttt::tc;

constexpr int BM = 128;                 // accumulator rows (TMEM lanes)
constexpr int BK = 64;                  // K elements per stage (one 128-byte swizzle row)
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int NUM_EPI_WARPS = 8;
constexpr int NTHREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int ACC_COLS = 256;           // per accumulator buffer

enum Kind { K_GATEUP = 0, K_VHAT = 1, K_GRAM = 2, K_APPLY = 3, K_INTRA = 4 };

// Per family: pipeline stages, bytes per stage, K elements per stage (KB), offset
// of the B operand inside a stage, and shared memory for the epilogue.
template <int FAM> struct Cfg;
template <> struct Cfg<FAM_ZV> {
  static constexpr int STAGES = 4, STAGE_BYTES = 48 * 1024, KB = 64, B_OFF = A_BYTES, EPI_BYTES = 0, NBUF = 2;
};
template <> struct Cfg<FAM_GRAM> {
  static constexpr int STAGES = 6, STAGE_BYTES = 32 * 1024, KB = 64, B_OFF = A_BYTES, EPI_BYTES = 0, NBUF = 2;
};
template <> struct Cfg<FAM_APPLY> {
  static constexpr int STAGES = 4, STAGE_BYTES = 48 * 1024, KB = 64, B_OFF = A_BYTES, EPI_BYTES = 0, NBUF = 2;
};
// 256 token rows per apply tile: two M=128 MMAs share every B stage, so a byte
// fetched from L2 feeds twice the flops; the two accumulators fill all of TMEM
// (no double buffering; the epilogue is short next to the K = d_ff mainloop).
// The epilogue stages O in one 32-row x 64-column box per warp and writes it with
// TMA stores (the stores leave while the next tile's MMAs run).
template <> struct Cfg<FAM_APPLY256> {
  static constexpr int STAGES = 3, STAGE_BYTES = 64 * 1024, KB = 64, B_OFF = 2 * A_BYTES,
                       EPI_BYTES = NUM_EPI_WARPS * 4096, NBUF = 1;
};
// Pair gate/up and target: CTA r of the cluster holds A rows m0 + 128 r .. of the
// 256-row tile and half of the N operand; 128 K per stage (two 64-wide boxes),
// 8 pair MMAs per stage.
template <> struct Cfg<FAM_ZV2> {
  static constexpr int STAGES = 3, STAGE_BYTES = 64 * 1024, KB = 128, B_OFF = 2 * A_BYTES, EPI_BYTES = 0,
                       NBUF = 2;
};
// Pair Gram: the ZZ^T and VV^T accumulators of a 256 x 256 block pair take all of
// TMEM (2 x 256 columns per CTA), so one accumulator set.
template <> struct Cfg<FAM_GRAM2> {
  static constexpr int STAGES = 3, STAGE_BYTES = 64 * 1024, KB = 128, B_OFF = 2 * A_BYTES, EPI_BYTES = 0,
                       NBUF = 1;
};
// Within-group products of the grouped scan: one 256 x 256 accumulator per group,
// two of them in TMEM (the epilogue of one overlaps the MMAs of the next).
template <> struct Cfg<FAM_PZ> {
  static constexpr int STAGES = 3, STAGE_BYTES = 64 * 1024, KB = 128, B_OFF = 2 * A_BYTES, EPI_BYTES = 0,
                       NBUF = 2;
};
template <int FAM> constexpr bool is_apply() { return FAM == FAM_APPLY || FAM == FAM_APPLY256; }
template <int FAM> constexpr bool is_zv() { return FAM == FAM_ZV || FAM == FAM_ZV2; }
template <int FAM> constexpr bool is_pair() { return FAM == FAM_ZV2 || FAM == FAM_GRAM2 || FAM == FAM_PZ; }
// token-block families: A and B rows both come from the tile's own tokens
template <int FAM> constexpr bool is_tokblk() { return FAM == FAM_GRAM || FAM == FAM_GRAM2 || FAM == FAM_PZ; }
template <int FAM> constexpr bool is_gram() { return FAM == FAM_GRAM || FAM == FAM_GRAM2; }

template <int FAM>
constexpr int smem_bytes() {
  return 1024 /*alignment slack*/ + Cfg<FAM>::STAGES * Cfg<FAM>::STAGE_BYTES + Cfg<FAM>::EPI_BYTES +
         256 /*barriers*/;
}
static_assert(smem_bytes<FAM_ZV>() <= 232448 && smem_bytes<FAM_APPLY256>() <= 232448, "kernel exceeds shared memory");

struct Job {
  int kind;
  int b;
  int m0, n0;     // tile origin: rows / columns of the accumulator in the operand index spaces
  int t0;         // first token of the tile's chunk (Gram, apply)
  int chunk;
  int pair;       // GRAM: tile pair index
  int nseg;
  int kb0[2], kb1[2];
  int acc_col[2];
  int n_mma;
  int nsrc;       // APPLY: 1 = W0 only, 2 = W0 and the state snapshot
  uint32_t tx;    // bytes per stage
  bool a_mn, b_mn;
  int halves;     // M=128 MMAs per K step (2: A holds 256 rows, accumulators 256 columns apart)
};

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------ decoding
template <int ROWS>
__device__ __forceinline__ void decode_zv(const TcParams& p, int tile, Job& j) {
  const int tiles_m = cdiv(p.T, ROWS);
  const int ncol = p.kind == K_GATEUP ? 128 : p.vn;  // gate/up: 128 gate + 128 up columns
  const int N = p.kind == K_GATEUP ? p.F : p.d;
  const int tiles_n = N / ncol;
  const int M_all = p.B * tiles_m;
  constexpr int G = 16;  // m-tiles per raster group
  const int per_group = G * tiles_n;
  const int g = tile / per_group, r = tile % per_group;
  const int m_first = g * G;
  const int gm = min(G, M_all - m_first);
  const int mm = m_first + r % gm;
  const int nt = r / gm;
  j.kind = p.kind;
  j.b = mm / tiles_m;
  j.m0 = (mm % tiles_m) * ROWS;
  j.n0 = nt * ncol;
  j.t0 = 0;
  j.chunk = 0;
  j.pair = 0;
  j.nseg = 1;
  j.kb0[0] = 0;
  j.kb1[0] = p.d / BK;
  j.acc_col[0] = 0;
  j.nsrc = 1;
  if (p.kind == K_GATEUP) {
    j.n_mma = 256;
    j.tx = ROWS * BK * 2 + 2 * 128 * BK * 2;
    j.a_mn = false;
    j.b_mn = false;
  } else {
    j.n_mma = p.vn;
    j.tx = A_BYTES + p.vn * BK * 2;
    j.a_mn = false;
    j.b_mn = true;
  }
  j.halves = ROWS == 256 ? 2 : 1;
}

__device__ __forceinline__ void decode_gram(const TcParams& p, int tile, Job& j) {
  const int per_row = p.k * p.npairs;
  j.kind = K_GRAM;
  j.b = tile / per_row;
  const int r = tile % per_row;
  j.chunk = r / p.npairs;
  j.pair = r % p.npairs;
  int ti = 0, rem = j.pair;
  while (rem >= p.ct - ti) { rem -= p.ct - ti; ++ti; }
  j.m0 = ti * p.tr;
  j.n0 = (ti + rem) * p.tr;
  j.t0 = j.chunk * p.C;
  j.nseg = 2;
  j.kb0[0] = 0; j.kb1[0] = p.F / BK; j.acc_col[0] = 0;     // Z Z^T
  j.kb0[1] = 0; j.kb1[1] = p.d / BK; j.acc_col[1] = 128;   // V V^T
  j.n_mma = 128;
  j.nsrc = 1;
  j.tx = 2 * p.tr * BK * 2;
  j.a_mn = false;
  j.b_mn = false;
}

template <int ROWS>  // 0: p.tr rows per tile; 256: two 128-row halves
__device__ __forceinline__ void decode_apply(const TcParams& p, int tile, Job& j) {
  const int rows = ROWS ? ROWS : p.tr;
  const int tiles_n = p.d / 128;
  const int tiles_m = p.C / rows;
  const int per_row = tiles_m * tiles_n;
  const int per_chunk = p.B * per_row;
  j.kind = K_APPLY;
  j.chunk = p.apply_chunk0 + tile / per_chunk;
  j.t0 = j.chunk * p.C;
  j.b = (tile % per_chunk) / per_row;
  // Row blocks vary fastest: the tiles that read one 128-column slice of the
  // chunk's snapshot (and of W0) are consecutive, so they run at the same time on
  // neighbouring CTAs and the slice comes from DRAM once.
  const int r = tile % per_row;
  j.m0 = (r % tiles_m) * rows;    // row offset inside the chunk
  j.n0 = (r / tiles_m) * 128;     // output column (d index)
  j.pair = 0;
  j.nseg = 1;
  j.acc_col[0] = 0;
  j.nsrc = p.meta[(size_t)j.b * p.k + j.chunk].cont ? 2 : 1;
  j.kb0[0] = 0;
  j.kb1[0] = p.F / BK;
  j.n_mma = 128 * j.nsrc;
  j.tx = rows * BK * 2 + j.nsrc * 128 * BK * 2;
  j.halves = ROWS == 256 ? 2 : 1;
  j.a_mn = false;
  j.b_mn = false;
}

template <int FAM>
__device__ __forceinline__ void decode(const TcParams& p, int tile, Job& j) {
  j.halves = 1;
  if constexpr (FAM == FAM_ZV) decode_zv<128>(p, tile, j);
  else if constexpr (FAM == FAM_ZV2) {
    // 256-row pair tile; each CTA moves its A half and its half of the N operand,
    // 128 K per stage; the leader's barrier counts both CTAs' bytes.
    decode_zv<256>(p, tile, j);
    j.halves = 1;
    // K: d; or, within-group term, the group's tokens up to the end of the tile's
    // 256-row block (P is zero beyond)
    j.kb1[0] = (p.kind == K_INTRA ? ((j.m0 % p.gl) / 256 + 1) * 256 : p.d) / 128;
    j.tx = 2 * (128 * 128 * 2 + (j.n_mma / 2) * 128 * 2);
  }
  else if constexpr (FAM == FAM_GRAM) decode_gram(p, tile, j);
  else if constexpr (FAM == FAM_GRAM2) {
    // p.tr = 256, p.ct = C / 256, p.npairs = ct (ct + 1) / 2; 128 K per stage
    decode_gram(p, tile, j);
    j.kb1[0] = p.F / 128;
    j.kb1[1] = p.d / 128;
    j.acc_col[1] = 256;
    j.n_mma = 256;
    j.tx = 2 * (2 * 128 * 128 * 2);
  }
  else if constexpr (FAM == FAM_PZ) {
    // one 256 x 256 block (row block rb, column block cb <= rb) of one group of
    // p.gl tokens of one row: its rows against its columns, K = d_ff
    const int groups = cdiv(p.T, p.gl);
    const int nb = p.gl / 256;
    const int per_group = nb * (nb + 1) / 2;
    const int g = tile / per_group;
    int rb = 0, rem = tile % per_group;
    while (rem > rb) { rem -= rb + 1; ++rb; }
    j.kind = K_GRAM;
    j.b = g / groups;
    j.t0 = (g % groups) * p.gl;
    j.m0 = rb * 256;
    j.n0 = rem * 256;
    j.chunk = j.pair = 0;
    j.nseg = 1;
    j.kb0[0] = 0;
    j.kb1[0] = p.F / 128;
    j.acc_col[0] = 0;
    j.n_mma = 256;
    j.nsrc = 1;
    j.tx = 2 * (2 * 128 * 128 * 2);
    j.a_mn = j.b_mn = false;
  }
  else if constexpr (FAM == FAM_APPLY) decode_apply<0>(p, tile, j);
  else decode_apply<256>(p, tile, j);
}

// i-th tile of this block (static round-robin schedule), or -1 past the end.
template <int FAM>
__device__ __forceinline__ int seq_tile(const TcParams& p, uint32_t i) {
  const long long w = is_pair<FAM>() ? (long long)cluster_id_x() : (long long)blockIdx.x;
  const long long nw = is_pair<FAM>() ? (long long)cluster_count_x() : (long long)gridDim.x;
  const long long t = w + (long long)i * nw;
  return t < p.n_tiles ? (int)t : -1;
}

// ------------------------------------------------------------------ producer
template <int FAM>
__device__ __forceinline__ void issue_loads(const TcParams& p, const Job& j, int seg, int kb, uint8_t* sa,
                                            uint8_t* sb, uint64_t* bar) {
  const int kx = kb * BK;
  if constexpr (is_pair<FAM>()) {
    // 128 K per stage: two 64-wide K boxes of this CTA's 128 A rows, then its half
    // of the N operand (gate rows on CTA 0, up rows on CTA 1; or target columns).
    const uint32_t r = cluster_rank();
    const uint32_t fb = map_to_rank(smem_u32(bar), 0);
    const int k0 = kb * 128;
    const int arow = (is_tokblk<FAM>() ? j.t0 : 0) + j.m0 + 128 * (int)r;
    const CUtensorMap* am = is_gram<FAM>() && seg == 1 ? &p.map[1] : &p.map[0];   // Gram: Z, then V
    tma_load_3d_pair(sa, am, fb, k0, arow, j.b);
    tma_load_3d_pair(sa + A_BYTES, am, fb, k0 + 64, arow, j.b);
    if constexpr (is_tokblk<FAM>()) {                               // rows of the other token block
      const int brow = j.t0 + j.n0 + 128 * (int)r;
      tma_load_3d_pair(sb, am, fb, k0, brow, j.b);
      tma_load_3d_pair(sb + 128 * BK * 2, am, fb, k0 + 64, brow, j.b);
    } else if (j.kind == K_GATEUP) {
      const CUtensorMap* wm = r == 0 ? &p.map[1] : &p.map[2];
      tma_load_3d_pair(sb, wm, fb, k0, j.n0, 0);
      tma_load_3d_pair(sb + 128 * BK * 2, wm, fb, k0 + 64, j.n0, 0);
    } else {
      // Wtarget[k][n] (or, within-group term, V'[b][group token k][n]), n contiguous
      const int nh = p.vn / 2;
      const bool intra = j.kind == K_INTRA;
      const int kofs = intra ? j.m0 - j.m0 % p.gl : 0;  // the group's first token
      for (int q = 0; q < nh / 64; ++q)
        tma_load_3d_pair(sb + q * 64 * 128 * 2, &p.map[1], fb, j.n0 + (int)r * nh + 64 * q, kofs + k0,
                         intra ? j.b : 0);
    }
  } else if constexpr (is_zv<FAM>()) {
    if (j.kind == K_GATEUP) {
      tma_load_3d(sa, &p.map[0], bar, kx, j.m0, j.b);              // H rows
      if (j.halves == 2) tma_load_3d(sa + A_BYTES, &p.map[0], bar, kx, j.m0 + 128, j.b);
      tma_load_3d(sb, &p.map[1], bar, kx, j.n0, 0);                   // Wgate rows
      tma_load_3d(sb + 128 * BK * 2, &p.map[2], bar, kx, j.n0, 0);    // Wup rows
    } else {
      tma_load_3d(sa, &p.map[0], bar, kx, j.m0, j.b);              // U rows
      for (int q = 0; q < p.vn / 64; ++q)                          // Wtarget[k][n], n contiguous
        tma_load_3d(sb + q * 64 * BK * 2, &p.map[1], bar, j.n0 + 64 * q, kx, 0);
    }
  } else if constexpr (FAM == FAM_GRAM) {
    const CUtensorMap* m = seg == 0 ? &p.map[0] : &p.map[1];       // Z or V
    tma_load_3d(sa, m, bar, kx, j.t0 + j.m0, j.b);
    tma_load_3d(sb, m, bar, kx, j.t0 + j.n0, j.b);
  } else if constexpr (is_apply<FAM>()) {
    tma_load_3d(sa, &p.map[0], bar, kx, j.t0 + j.m0, j.b);        // Z rows of the chunk
    if (j.halves == 2) tma_load_3d(sa + A_BYTES, &p.map[0], bar, kx, j.t0 + j.m0 + 128, j.b);
    // W0 (d F bf16, read by every tile of the launch) stays in L2; a snapshot slice
    // is read by the chunk's row-block tiles at once, then never again
    tma_load_3d_hint(sb, &p.map[1], bar, kx, j.n0, 0, l2_policy_evict_last());        // Wdown0 rows
    if (j.nsrc == 2)
      tma_load_3d_hint(sb + 128 * BK * 2, &p.map[2], bar, kx, j.n0, (j.chunk % p.nslots) * p.B + j.b,
                       l2_policy_evict_first());                                     // S_i rows
  }
}

// ------------------------------------------------------------------ epilogues
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void st_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = w;
  }
}

// Named barrier among the epilogue warps only.
__device__ __forceinline__ void epi_sync() {
  __syncwarp();
  asm volatile("bar.sync 1, %0;" ::"n"(NUM_EPI_WARPS * 32) : "memory");
}

template <int FAM>
__device__ __forceinline__ void epilogue_tile(const TcParams& p, const Job& j, uint32_t tacc, int half, int row,
                                              int lane, int ew, float* red, uint8_t* ebox, int& nst) {
  uint32_t r0[32], r1[32];
  float v[32];
  if constexpr (is_zv<FAM>()) {
    // Two M halves (256-row gate/up tiles): this warp drains rows 128 half .. of
    // all 128 output columns, from the accumulator 256 TMEM columns further up.
    const bool two = j.halves == 2;
    if (two) tacc += half * 256;
    const int t = j.m0 + (two ? half * 128 : 0) + row;
    const bool valid = t < p.T;
    if (j.kind == K_GATEUP) {
      __nv_bfloat16* zrow = reinterpret_cast<__nv_bfloat16*>(p.out0) + ((size_t)j.b * p.T + t) * p.F + j.n0;
      const int c0 = two ? 0 : half * 64, c1 = two ? 128 : half * 64 + 64;
#pragma unroll 1
      for (int c = c0; c < c1; c += 32) {
        tmem_ld32(tacc + c, r0);
        tmem_ld32(tacc + 128 + c, r1);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = silu_fast(__uint_as_float(r0[i])) * __uint_as_float(r1[i]);
        if (valid) st_bf16x32(zrow + c, v);
      }
    } else {
      const int chunk = t / p.C;
      // the target keeps the rows of each chunk's last document segment; the
      // within-group term keeps every row
      const bool keep = valid && (j.kind == K_INTRA || t >= p.meta[(size_t)j.b * p.k + min(chunk, p.k - 1)].last_start);
      __nv_bfloat16* vrow = reinterpret_cast<__nv_bfloat16*>(p.out0) + ((size_t)j.b * p.T + t) * p.d + j.n0;
      const int w = p.vn / 2;  // columns drained by this warp
#pragma unroll 1
      for (int c = half * w; c < half * w + w; c += 32) {
        tmem_ld32(tacc + c, r0);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = keep ? __uint_as_float(r0[i]) : 0.0f;
        if (valid) st_bf16x32(vrow + c, v);
      }
    }
  } else if constexpr (FAM == FAM_PZ) {
    // Row t of the group (j.m0: the row block and this CTA's offset) against
    // columns u of the column block j.n0, [128 half, 128 half + 128): z_t . z_u is
    // kept where u lies in t's document (u >= lo(t)) and in an earlier chunk (u <
    // the start of t's chunk).
    const int t = j.t0 + j.m0 + row;
    const bool valid = t < p.T;
    const int lo = valid ? j.t0 + (int)p.glo[(size_t)j.b * p.T + t] : 0;
    const int hi = valid ? (t / p.cs) * p.cs : 0;
    __nv_bfloat16* prow = reinterpret_cast<__nv_bfloat16*>(p.out0) + ((size_t)j.b * p.T + t) * p.gl + j.n0;
#pragma unroll 1
    for (int c = half * 128; c < half * 128 + 128; c += 32) {
      tmem_ld32(tacc + c, r0);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int u = j.t0 + j.n0 + c + i;
        v[i] = (u >= lo && u < hi) ? __uint_as_float(r0[i]) : 0.0f;
      }
      if (valid) st_bf16x32(prow + c, v);
    }
  } else if constexpr (FAM == FAM_GRAM2) {
    // This CTA's 128 rows of the 256 x 256 block pair; warp half h sums columns
    // [128 h, 128 h + 128) of (Z Z^T) * (V V^T).  Diagonal pairs count once, the
    // others twice (the mirrored pair is not computed).
    float s = 0.0f;
#pragma unroll 1
    for (int c = half * 128; c < half * 128 + 128; c += 32) {
      tmem_ld32(tacc + c, r0);
      tmem_ld32(tacc + 256 + c, r1);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) s = fmaf(__uint_as_float(r0[i]), __uint_as_float(r1[i]), s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[ew] = s;
    epi_sync();
    if (ew == 0 && lane == 0) {
      float tot = 0.0f;
      for (int w = 0; w < NUM_EPI_WARPS; ++w) tot += red[w];
      const float wgt = (j.m0 / 256) == (j.n0 / 256) ? 1.0f : 2.0f;
      p.partials[(((size_t)j.b * p.k + j.chunk) * p.npairs + j.pair) * 2 + cluster_rank()] = wgt * tot;
    }
    epi_sync();
  } else if constexpr (FAM == FAM_GRAM) {
    // Only rows and columns below tr hold Gram entries of this tile pair.
    float s = 0.0f;
#pragma unroll 1
    for (int c = half * 64; c < half * 64 + 64; c += 32) {
      if (c >= p.tr) break;  // warp-uniform
      tmem_ld32(tacc + c, r0);
      tmem_ld32(tacc + 128 + c, r1);
      tmem_ld_wait();
      if (row < p.tr) {
#pragma unroll
        for (int i = 0; i < 32; ++i) s = fmaf(__uint_as_float(r0[i]), __uint_as_float(r1[i]), s);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[ew] = s;
    epi_sync();
    if (ew == 0 && lane == 0) {
      float tot = 0.0f;
      for (int w = 0; w < NUM_EPI_WARPS; ++w) tot += red[w];
      const float wgt = j.m0 == j.n0 ? 1.0f : 2.0f;
      p.partials[((size_t)j.b * p.k + j.chunk) * p.npairs + j.pair] = wgt * tot;
    }
    epi_sync();
  } else if constexpr (is_apply<FAM>()) {
    // FAM_APPLY: this warp drains columns [64 half, 64 half + 64) of a 128-row tile;
    // FAM_APPLY256: all 128 columns of rows 128 half .. of a 256-row tile, whose
    // accumulator sits 256 TMEM columns further for the upper half.
    constexpr bool two = FAM == FAM_APPLY256;
    const int row_in_tile = two ? half * 128 + row : row;
    if (two) tacc += half * 256;
    const int c_begin = two ? 0 : half * 64, c_end = two ? 128 : half * 64 + 64;
    const ChunkMeta m = p.meta[(size_t)j.b * p.k + j.chunk];
    const int t = j.t0 + j.m0 + row_in_tile;
    const bool valid = (two || row < p.tr) && t < p.T;
    const bool carry = j.nsrc == 2 && m.cont && t < m.first_end;
    const bool tma_o = two && p.o_tma;
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out0) + ((size_t)j.b * p.T + t) * p.d + j.n0;
    const __nv_bfloat16* hrow =
        p.resid ? reinterpret_cast<const __nv_bfloat16*>(p.resid) + ((size_t)j.b * p.T + t) * p.d + j.n0 : nullptr;
    float* drow = p.out1 ? p.out1 + ((size_t)j.b * p.T + t) * p.d + j.n0 : nullptr;
    const __nv_bfloat16* erow =
        p.intra ? reinterpret_cast<const __nv_bfloat16*>(p.intra) + ((size_t)j.b * p.T + t) * p.d + j.n0 : nullptr;
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 32) {
      // the row's E and H words are requested before the accumulator is read, so
      // their latency overlaps the TMEM round trip
      uint4 ev4[4], hv4[4];
      if (erow && valid) {
#pragma unroll
        for (int q = 0; q < 4; ++q) ev4[q] = reinterpret_cast<const uint4*>(erow + c)[q];
      }
      if (hrow && valid) {
#pragma unroll
        for (int q = 0; q < 4; ++q) hv4[q] = reinterpret_cast<const uint4*>(hrow + c)[q];
      }
      tmem_ld32(tacc + c, r0);
      if (j.nsrc == 2) tmem_ld32(tacc + 128 + c, r1);
      tmem_ld_wait();
      float e[32];
      if (erow && valid) {
        // the grouped scan's within-group term joins the fast-weight part
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 ev = ev4[q];
          const uint32_t ew4[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&ew4[x]);
            e[8 * q + 2 * x] = __low2float(h2);
            e[8 * q + 2 * x + 1] = __high2float(h2);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) e[i] = 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float dv = (carry ? __uint_as_float(r1[i]) : 0.0f) + e[i];
        v[i] = __uint_as_float(r0[i]) + dv;
        r1[i] = __float_as_uint(dv);
      }
      if (valid) {
        if (hrow) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 hv = hv4[q];
            const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&hw[e]);
              v[8 * q + 2 * e] += __low2float(h2);
              v[8 * q + 2 * e + 1] += __high2float(h2);
            }
          }
        }
        if (!tma_o) st_bf16x32(orow + c, v);
        if (drow) {
          float4* d4 = reinterpret_cast<float4*>(drow + c);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            d4[q] = make_float4(__uint_as_float(r1[4 * q]), __uint_as_float(r1[4 * q + 1]),
                                __uint_as_float(r1[4 * q + 2]), __uint_as_float(r1[4 * q + 3]));
        }
      }
      if (tma_o) {
        // 32 columns into the warp's box (128-byte swizzled rows); once the box holds
        // 64 columns it goes out by TMA (rows past T are clipped by the tensor map)
        if ((c & 63) == 0 && nst > 0) {
          if (lane == 0) bulk_wait_read<0>();  // the box's previous store has read it
          __syncwarp();
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = ((c & 63) >> 3) + q;
          *reinterpret_cast<uint4*>(ebox + lane * 128 + ((e ^ (lane & 7)) << 4)) =
              make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                         pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
        }
        if ((c & 63) == 32) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&p.map[6], ebox, j.n0 + (c & ~63), j.t0 + j.m0 + half * 128 + (row - lane), j.b);
            bulk_commit();
          }
          ++nst;
        }
      }
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int FAM>
__global__ void __launch_bounds__(NTHREADS, 1) tc_kernel(const __grid_constant__ TcParams p) {
  constexpr int STAGES = Cfg<FAM>::STAGES;
  constexpr int STAGE_BYTES = Cfg<FAM>::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* epi = smem + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi + Cfg<FAM>::EPI_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* counters = reinterpret_cast<uint32_t*>(tmem_slot + 2);  // [0] issued, [1] consumed
  float* red = reinterpret_cast<float*>(tmem_slot + 5);              // NUM_EPI_WARPS floats

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr bool PAIR = is_pair<FAM>();
  const uint32_t rank = PAIR ? cluster_rank() : 0u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], NUM_EPI_WARPS * (PAIR ? 2 : 1));
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    counters[0] = counters[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    const int nmaps = is_apply<FAM>() ? 3 : FAM == FAM_PZ ? 1 : (is_gram<FAM>() ? 2 : (p.kind == K_GATEUP ? 3 : 2));
    for (int i = 0; i < nmaps; ++i) prefetch_tmap(&p.map[i]);
    if (FAM == FAM_APPLY256 && p.o_tma) prefetch_tmap(&p.map[6]);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, 2 * ACC_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 2 * ACC_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t i = 0; ok; ++i) {
        const int tile = seq_tile<FAM>(p, i);
        if (tile < 0) break;
        Job j;
        decode<FAM>(p, tile, j);
        for (int seg = 0; seg < j.nseg && ok; ++seg) {
          for (int kb = j.kb0[seg]; kb < j.kb1[seg]; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait_or_abort(&empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
            uint8_t* sa = stages + s * STAGE_BYTES;
            if (!PAIR || rank == 0) mbar_arrive_expect_tx(&full[s], j.tx);
            issue_loads<FAM>(p, j, seg, kb, sa, sa + Cfg<FAM>::B_OFF, &full[s]);
          }
        }
      }
      if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
      counters[0] = it;
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      bool ready = mbar_try_wait(&full[0], 0);
      for (uint32_t i = 0; ok; ++i, ++tcount) {
        const int tile = seq_tile<FAM>(p, i);
        if (tile < 0) break;
        Job j;
        decode<FAM>(p, tile, j);
        const int buf = Cfg<FAM>::NBUF == 2 ? (tcount & 1) : 0;
        const uint32_t aph = Cfg<FAM>::NBUF == 2 ? ((tcount >> 1) & 1) : (tcount & 1);
        const bool got = PAIR ? mbar_wait_cluster(&acc_empty[buf], aph ^ 1)
                              : mbar_wait_or_abort(&acc_empty[buf], aph ^ 1, abort_flag);
        if (!got || (PAIR && *abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tacc = tmem_base + buf * ACC_COLS;
        const uint32_t idesc = idesc_bf16(PAIR ? 256 : BM, j.n_mma, j.a_mn, j.b_mn);
        for (int seg = 0; seg < j.nseg && ok; ++seg) {
          for (int kb = j.kb0[seg]; kb < j.kb1[seg]; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!ready && !mbar_wait_or_abort(&full[s], ph, abort_flag)) { ok = false; break; }
            // peek at the next stage while this one's MMAs are queued
            ready = mbar_try_wait(&full[(it + 1) % STAGES], ((it + 1) / STAGES) & 1);
            const uint32_t a_addr = smem_u32(stages + s * STAGE_BYTES);
            const uint32_t b_addr = a_addr + Cfg<FAM>::B_OFF;
            constexpr int KB = Cfg<FAM>::KB;
#pragma unroll
            for (int ks = 0; ks < KB / 16; ++ks) {
              // MN-major: 16 K rows of 128 B per step, MN blocks KB rows apart.
              // K-major: 32 B per step inside a 64-wide K box; boxes of 128 rows
              // (16 KB) follow each other when a stage holds 128 K.
              const uint32_t kofs = (ks / 4) * 16384 + (ks % 4) * 32;
              const uint64_t ad = j.a_mn ? sdesc_sw128(a_addr + ks * 2048, KB * 128, 1024)
                                         : sdesc_sw128(a_addr + kofs, 16, 1024);
              const uint64_t bd = j.b_mn ? sdesc_sw128(b_addr + ks * 2048, KB * 128, 1024)
                                         : sdesc_sw128(b_addr + kofs, 16, 1024);
              const uint32_t acc_flag = (kb > j.kb0[seg] || ks > 0) ? 1u : 0u;
              if constexpr (PAIR) {
                mma_bf16_pair(tacc + j.acc_col[seg], ad, bd, idesc, acc_flag);
                continue;
              }
              mma_bf16(tacc + j.acc_col[seg], ad, bd, idesc, acc_flag);
              if (j.halves == 2)  // rows 128..255 of A (K-major, 16 KB further), next 256 columns
                mma_bf16(tacc + 256 + j.acc_col[seg], sdesc_sw128(a_addr + A_BYTES + ks * 32, 16, 1024), bd,
                         idesc, acc_flag);
            }
            if constexpr (PAIR) mma_commit_pair(&empty[s], 3); else mma_commit(&empty[s]);
          }
        }
        if (ok) {
          if constexpr (PAIR) mma_commit_pair(&acc_full[buf], 3); else mma_commit(&acc_full[buf]);
        }
      }
      if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
      counters[1] = it;
      // Let every MMA issued by this thread finish before TMEM is released.
      if constexpr (PAIR) mma_commit_pair(drain, 1); else mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    const int ew = warp - 2;
    const int quarter = warp & 3;      // TMEM lanes this warp may access
    const int half = ew >> 2;          // which half of the columns this warp drains
    const int row = quarter * 32 + lane;
    uint32_t tcount = 0;
    bool ok = true;
    int nst = 0;  // O boxes this warp has stored (256-row apply)
    const uint32_t empty0 = PAIR ? map_to_rank(smem_u32(acc_empty), 0) : 0u;  // the leader's acc_empty[0]
    for (uint32_t i = 0;; ++i, ++tcount) {
      const int tile = seq_tile<FAM>(p, i);
      if (tile < 0) break;
      Job j;
      decode<FAM>(p, tile, j);
      const int buf = Cfg<FAM>::NBUF == 2 ? (tcount & 1) : 0;
      const uint32_t aph = Cfg<FAM>::NBUF == 2 ? ((tcount >> 1) & 1) : (tcount & 1);
      // Every epilogue warp leaves only through this wait (all of them wait on the
      // same phases), so none is left behind at the epilogue's named barrier.
      if (!mbar_wait(&acc_full[buf], aph)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * ACC_COLS + ((uint32_t)(quarter * 32) << 16);
      if constexpr (PAIR) j.m0 += 128 * (int)rank;  // this CTA's rows of the pair tile
      epilogue_tile<FAM>(p, j, tacc, half, row, lane, ew, red, epi + ew * 4096, nst);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(empty0 + 8u * buf);
        else mbar_arrive(&acc_empty[buf]);
      }
      if constexpr (is_apply<FAM>()) {
        // while the next tile's MMAs run, bring this thread's rows of its
        // within-group term and residual into L2
        if (p.intra || p.resid) {
          const int nt = seq_tile<FAM>(p, i + 1);
          if (nt >= 0) {
            Job jn;
            decode<FAM>(p, nt, jn);
            const int rin = FAM == FAM_APPLY256 ? half * 128 + row : row;
            const int tn = jn.t0 + jn.m0 + rin;
            if (tn < p.T && (FAM == FAM_APPLY256 || row < p.tr)) {
              const size_t off = ((size_t)jn.b * p.T + tn) * p.d + jn.n0 + (FAM == FAM_APPLY256 ? 0 : half * 64);
              const int bytes = FAM == FAM_APPLY256 ? 256 : 128;
              for (int q = 0; q < bytes; q += 128) {
                if (p.intra) prefetch_l2(reinterpret_cast<const uint8_t*>(p.intra) + off * 2 + q);
                if (p.resid) prefetch_l2(reinterpret_cast<const uint8_t*>(p.resid) + off * 2 + q);
              }
            }
          }
        }
      }
    }
    if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
    if (lane == 0) bulk_wait<0>();
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && rank == 0) {
    // Wait (bounded) for copies that were issued but never consumed, so no TMA
    // write lands in shared memory after the block has exited.
    for (uint32_t it = counters[1]; it < counters[0]; ++it)
      mbar_wait(&full[it % STAGES], (it / STAGES) & 1);
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, 2 * ACC_COLS);
    else tmem_dealloc(tmem_base, 2 * ACC_COLS);
  }
}

// ------------------------------------------------------------------ state update
// S_{c+1} = keep_c S_c + alpha_c eta V_c^T Z_c for the chunks c of one launch.
// V arrives pre-scaled by alpha_c eta per row.  The MMAs form each chunk's delta
// from zero in one of two TMEM slots (256 fp32 columns each, taken in turn chunk
// by chunk), so the tensor cores never add a small delta onto a large running
// sum.  The fp32 state of the worker's current tile lives in the registers of
// the epilogue warps (one TMEM lane row, 128 columns per thread) and takes each
// delta with an ordinary fp32 add, rounded to nearest.  While the epilogue folds
// chunk c's delta and writes the bf16 snapshot of S_{c+1} for the apply, the MMAs
// of chunk c+1 fill the other slot.  A chunk holding a document start drops the
// carried state before its delta is added.  A tile's fp32 state comes in from HBM
// before its first chunk of the launch and goes back after its last.
//
// Two forms of one kernel body:
//   PAIR = false: one CTA per 128 (d) x 256 (F) state tile, M=128 MMAs.
//   PAIR = true : a cluster of two CTAs per 256 x 256 tile, M=256 pair MMAs
//                 (cta_group::2).  CTA r holds d rows m0 + 128 r .. +127 of the
//                 tile in its TMEM and loads those V columns and Z columns
//                 n0 + 128 r .. +127 per stage; the even CTA issues the MMAs.  Per
//                 FLOP this moves 2/3 of the operand bytes of the single-CTA form.
constexpr int UPD_BOX_BYTES = 32 * 128;               // a warp's 32-row x 64-column snapshot box
// Three warpgroups: warps 0-7 the epilogue (each thread holds 128 fp32 state
// values), warp 8 the TMA producer, warp 9 the MMA issuer, warps 10-11 idle.
// Twelve warps put three on each SM sub-partition, which caps a thread at 168
// registers at launch; the third warpgroup then drops to UPD_REGS_LOW and the two
// epilogue warpgroups rise to UPD_REGS_EPI, an exact trade:
// 128 x (168 - 56) = 256 x (224 - 168).  The launcher checks that the kernel was
// compiled to 168 registers, the count this balance assumes.
constexpr int UPD_THREADS = 384;
constexpr int UPD_WARP_TMA = 8, UPD_WARP_MMA = 9;
constexpr int UPD_REGS_LAUNCH = 168, UPD_REGS_LOW = 56, UPD_REGS_EPI = 224;
static_assert((UPD_THREADS - 32 * NUM_EPI_WARPS) * (UPD_REGS_LAUNCH - UPD_REGS_LOW) ==
                  32 * NUM_EPI_WARPS * (UPD_REGS_EPI - UPD_REGS_LAUNCH),
              "the register trade of the update kernel must balance");

// KB tokens per stage: 128 (8 MMAs per stage; the per-stage issue overhead is
// paid half as often) when the chunk length is a multiple of 128, else 64 (a
// stage never straddles two chunks).  BOXES snapshot boxes per warp: with two,
// a box store stays in flight while the next box is filled.
template <bool PAIR, int KB> struct UpdCfg {
  static constexpr int STAGES = KB == 128 ? (PAIR ? 3 : 2) : (PAIR ? 5 : 3);
  static constexpr int BOXES = KB == 128 ? 1 : 2;
  static constexpr int A_BYTES = 128 * KB * 2;                            // V: 128 d columns
  static constexpr int B_COLS = PAIR ? 128 : 256;                         // Z columns this CTA loads
  static constexpr int STAGE_BYTES = A_BYTES + B_COLS * KB * 2;
  static constexpr int TILE_ROWS = PAIR ? 256 : 128;                      // d rows per state tile
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + NUM_EPI_WARPS * BOXES * UPD_BOX_BYTES + 256;
};
static_assert(UpdCfg<false, 64>::SMEM <= 232448 && UpdCfg<true, 64>::SMEM <= 232448 &&
                  UpdCfg<false, 128>::SMEM <= 232448 && UpdCfg<true, 128>::SMEM <= 232448,
              "update kernel exceeds shared memory");

struct UpdJob {
  int X;      // state tile: (b, nt2, mt) of B x ceil(F/256) x (d/TILE_ROWS), mt fastest
  int c;      // chunk of the launch, 0 .. dchunks-1
  int chunk;  // absolute chunk index
  int b, m0, n0;
};

// Job i of worker w (a CTA, or a CTA pair) of nw, or false past the end.  The
// worker's tiles are X_m = w + m nw; each is walked through every chunk of the
// launch before the next.  The delta of job i goes to TMEM slot i % 2.
template <bool PAIR, bool REV = false>
__device__ __forceinline__ bool upd_job(const TcParams& p, uint32_t i, int w, int nw, UpdJob& jb) {
  const uint32_t D = (uint32_t)p.dchunks;
  const long long X = (long long)w + (long long)(i / D) * nw;
  if (X >= p.n_tiles) return false;
  jb.X = (int)X;
  jb.c = (int)(i % D);
  jb.chunk = REV ? p.chunk + (int)D - 1 - jb.c : p.chunk + jb.c;  // REV: the chunks from the last
  // Row blocks vary fastest: the tiles in flight at one time (one per worker)
  // then cover few column blocks, so each chunk's Z columns come from DRAM about
  // once per launch (V, four times smaller, once per round of tiles).
  const int nt2s = (p.F + 255) / 256;
  const int mts = p.d / (PAIR ? 256 : 128);
  const int per_row = mts * nt2s;
  jb.b = jb.X / per_row;
  const int r = jb.X % per_row;
  jb.m0 = (r % mts) * (PAIR ? 256 : 128);
  jb.n0 = (r / mts) * 256;
  return true;
}

// K blocks of a chunk's delta: the forward's rows from the last segment's start;
// the reverse scan's the continued first segment (gO_F is zero outside it; a chunk
// without one still takes one block, of zeros, so its slot gets a delta).
template <bool REV, int UKB>
__device__ __forceinline__ void upd_kb_range(const TcParams& p, const ChunkMeta& m, int t0, int& kb0, int& kb1) {
  if (REV) {
    kb0 = 0;
    kb1 = m.cont ? max(1, cdiv(min(m.first_end, p.T) - t0, UKB)) : 1;
  } else {
    kb0 = (m.last_start - t0) / UKB;
    kb1 = cdiv(min(p.C, p.T - t0), UKB);
  }
}

// fp32 state, 128 x 128 blocked tiles; tile column block h of the 128-row block
// starting at d row m0 (a multiple of 128).  Inside a block, element (row, c) sits
// at float4 index (c / 4) * 128 + row, so a warp holding 32 consecutive rows moves
// 512 contiguous bytes per float4 column.
__device__ __forceinline__ float4* upd_state_block(const TcParams& p, int b, int m0, int n0, int h) {
  return reinterpret_cast<float4*>(p.S + (size_t)b * p.d * p.F +
                                   ((size_t)(m0 / 128) * (p.F / 128) + n0 / 128 + h) * (128 * 128));
}

// DELTA: also write each chunk's raw delta (the forward run for the backward); a
// separate build, so the forward's own update carries none of that code.
// REV: the reverse scan of the backward, G_i = keep_i G_{i+1} + gO_F^T Z_F from the
// last chunk down (A operand gO_F in place of V, rows of the continued first
// segment); each chunk's slot i receives bf16(G_{i+1}), the state before the chunk.
template <bool PAIR, int KB, bool DELTA, bool REV>
__global__ void __launch_bounds__(UPD_THREADS, 1) upd_kernel(const __grid_constant__ TcParams p) {
  using Cf = UpdCfg<PAIR, KB>;
  constexpr int STAGES = Cf::STAGES;
  constexpr int UPD_KB = KB;
  constexpr int UPD_BOXES = Cf::BOXES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* boxes = smem + STAGES * Cf::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(boxes + NUM_EPI_WARPS * UPD_BOXES * UPD_BOX_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* slot_free = empty + STAGES;  // [2] epilogue -> MMA: the slot's delta has been read
  uint64_t* slot_full = slot_free + 2;   // [2] MMA -> epilogue: the chunk's delta is complete
  uint64_t* drain = slot_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* counters = reinterpret_cast<uint32_t*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const int wk = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;      // worker (pair) index
  const int nwk = PAIR ? (int)cluster_count_x() : (int)gridDim.x;
  const int rofs = PAIR ? 128 * (int)rank : 0;                      // this CTA's rows / Z columns in the tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&slot_free[s], NUM_EPI_WARPS * (PAIR ? 2 : 1));
      mbar_init(&slot_full[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    counters[0] = counters[1] = 0;
    fence_mbar_init();
  }
  if (warp == UPD_WARP_TMA && lane == 0) {
    prefetch_tmap(&p.map[3]);
    prefetch_tmap(&p.map[4]);
    prefetch_tmap(&p.map[5]);
    if (DELTA) prefetch_tmap(&p.map[7]);
  }
  if (warp == UPD_WARP_MMA) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, 2 * ACC_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 2 * ACC_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < NUM_EPI_WARPS) {
    // the epilogue warpgroups take the registers the third warpgroup gives up
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(UPD_REGS_EPI));
    const int ew = warp;
    const int quarter = warp & 3;   // TMEM lanes this warp may access
    const int half = ew >> 2;       // 128-column half of the 256-column state tile
    const int row = quarter * 32 + lane;
    uint8_t* wboxes = boxes + ew * UPD_BOXES * UPD_BOX_BYTES;
    bool ok = true;
    int stores = 0;
    const uint32_t free0 = PAIR ? map_to_rank(smem_u32(slot_free), 0) : 0u;  // the leader's slot_free[0]
    // This thread's row of the current tile's state: columns 128 half .. +127.
    float st[128];
#pragma unroll
    for (int e = 0; e < 128; ++e) st[e] = 0.0f;

    UpdJob jb;
    for (uint32_t i = 0; upd_job<PAIR, REV>(p, i, wk, nwk, jb); ++i) {
      const int sl = (int)(i & 1);
      const ChunkMeta m = p.meta[(size_t)jb.b * p.k + jb.chunk];
      const int m0c = jb.m0 + rofs;
      const bool cols = jb.n0 + 128 * half < p.F;  // this warp's half lies inside the state
      // what the delta is added to: nothing (a document starts in the chunk: the
      // carried state is dropped), the state in registers, or (the tile's first
      // chunk of the launch) the state as the previous launch or the caller left it
      const float* sf = reinterpret_cast<const float*>(upd_state_block(p, jb.b, m0c, jb.n0, half));
      if constexpr (REV) {
        // the reverse scan stores the state before the chunk: bring in the start state first
        if (jb.c == 0 && jb.n0 + 128 * half < p.F) {
#pragma unroll
          for (int q = 0; q < 128; ++q) st[q] = sf[((q / 4) * 128 + row) * 4 + (q & 3)];
        }
      }
      const int base = m.has_start ? 0 : ((!REV && jb.c == 0) ? 2 : 1);
      const bool snap = REV || jb.chunk + 1 < p.k;
      const int slot = REV ? jb.chunk % p.nslots : (jb.chunk + 1) % p.nslots;
      // Folds 64 columns of the delta (one 64-column TMEM load) into st[64 hb ..].
      // the chunk's clip factor times eta, when V was not pre-scaled by it
      const float sc = p.upd_scale ? p.alpha[(size_t)jb.b * p.k + jb.chunk] * p.eta : 1.0f;
      auto fold = [&](const int hb, const uint32_t (&ra)[64]) {
#pragma unroll
        for (int q = 0; q < 64; ++q) {
          const int c = 64 * hb + q;
          const float old = base == 2 ? sf[((c / 4) * 128 + row) * 4 + (c & 3)] : base == 1 ? st[c] : 0.0f;
          st[c] = fmaf(sc, __uint_as_float(ra[q]), old);
        }
      };
      // Snapshot box hb: 32 rows x 64 columns of bf16(S_{chunk+1}) (what the apply of
      // chunk+1 reads), 128-byte swizzled, stored by TMA.
      auto store_box = [&](const int hb) {
        // boxes in turn (with the deltas' boxes in between when DELTA)
        uint8_t* box = wboxes + ((DELTA ? stores : hb) % UPD_BOXES) * UPD_BOX_BYTES;
        if (stores > 0) {
          // the store issued from this buffer UPD_BOXES boxes ago has read it
          if (lane == 0) bulk_wait_read<UPD_BOXES - 1>();
          __syncwarp();
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = 64 * hb + 8 * e;
          *reinterpret_cast<uint4*>(box + lane * 128 + ((e ^ (lane & 7)) << 4)) =
              make_uint4(pack_bf16(st[c], st[c + 1]), pack_bf16(st[c + 2], st[c + 3]),
                         pack_bf16(st[c + 4], st[c + 5]), pack_bf16(st[c + 6], st[c + 7]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // the snapshots (2 d F bytes per chunk, read back only by a later launch)
          // leave L2 first, so the chunk's V and Z, which every pair reads, stay there
          tma_store_3d_hint(&p.map[5], box, jb.n0 + 128 * half + 64 * hb, m0c + 32 * quarter,
                            slot * p.B + jb.b, l2_policy_evict_first());
          bulk_commit();
        }
        ++stores;
      };
      // For the backward: box hb of the chunk's raw delta V_L^T Z_L (the TMEM values
      // before alpha eta), bf16, into the chunk's [d][F] matrix of map[7].
      auto store_delta = [&](const int hb, const uint32_t (&ra)[64]) {
        uint8_t* box = wboxes + (stores % UPD_BOXES) * UPD_BOX_BYTES;
        if (stores > 0) {
          if (lane == 0) bulk_wait_read<UPD_BOXES - 1>();
          __syncwarp();
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<uint4*>(box + lane * 128 + ((e ^ (lane & 7)) << 4)) = make_uint4(
              pack_bf16(__uint_as_float(ra[8 * e]), __uint_as_float(ra[8 * e + 1])),
              pack_bf16(__uint_as_float(ra[8 * e + 2]), __uint_as_float(ra[8 * e + 3])),
              pack_bf16(__uint_as_float(ra[8 * e + 4]), __uint_as_float(ra[8 * e + 5])),
              pack_bf16(__uint_as_float(ra[8 * e + 6]), __uint_as_float(ra[8 * e + 7])));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&p.map[7], box, jb.n0 + 128 * half + 64 * hb, m0c + 32 * quarter, jb.chunk * p.B + jb.b);
          bulk_commit();
        }
        ++stores;
      };
      if (!mbar_wait(&slot_full[sl], (i >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      // Two halves of the warp's 128 columns, one 64-column TMEM load each: the
      // second half's load is in flight while the first is folded and stored.
      uint32_t x0[64], y0[64];
      const uint32_t tcol = tmem_base + sl * ACC_COLS + ((uint32_t)(quarter * 32) << 16) + 128 * half;
      if (cols) {
        tmem_ld64(tcol, x0);
        tmem_ld_wait();
        if constexpr (DELTA) store_delta(0, x0);
        if (REV && snap) store_box(0);
        fold(0, x0);
        tmem_ld64(tcol + 64, y0);
        if (!REV && snap) store_box(0);
        tmem_ld_wait();
      }
      // the slot's delta is in registers: the MMAs may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(free0 + 8u * sl);
        else mbar_arrive(&slot_free[sl]);
      }
      if (!cols) continue;
      if constexpr (DELTA) store_delta(1, y0);
      if (REV && snap) store_box(1);
      fold(1, y0);
      if (!REV && snap) store_box(1);
      if (jb.c == p.dchunks - 1) {
        // the tile's last chunk of the launch: the fp32 state goes back to HBM
        float4* dst = upd_state_block(p, jb.b, m0c, jb.n0, half);
        float* df = reinterpret_cast<float*>(dst);
#pragma unroll
        for (int q = 0; q < 128; ++q) df[((q / 4) * 128 + row) * 4 + (q & 3)] = st[q];
      }
    }
    if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
    if (lane == 0) bulk_wait<0>();
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(UPD_REGS_LOW));
    if (warp == UPD_WARP_TMA) {
      if (lane == 0) {
        uint32_t it = 0;
        bool ok = true;
        UpdJob jb;
        const uint32_t full0 = PAIR ? map_to_rank(smem_u32(full), 0) : 0u;  // the leader's full[0]
        // The next job's chunk metadata is requested one job ahead, so its round
        // trip never stands between two chunks' loads.
        bool have = upd_job<PAIR, REV>(p, 0, wk, nwk, jb);
        ChunkMeta m{};
        if (have) m = p.meta[(size_t)jb.b * p.k + jb.chunk];
        for (uint32_t i = 0; ok && have; ++i) {
          UpdJob jn;
          const bool hn = upd_job<PAIR, REV>(p, i + 1, wk, nwk, jn);
          ChunkMeta mn{};
          if (hn) mn = p.meta[(size_t)jn.b * p.k + jn.chunk];
          const int t0 = jb.chunk * p.C;
          int kb0, kb1;
          upd_kb_range<REV, UPD_KB>(p, m, t0, kb0, kb1);
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(&empty[s], ph ^ 1) || *abort_flag) { ok = false; break; }
            uint8_t* sa = stages + s * Cf::STAGE_BYTES;
            uint8_t* sb = sa + Cf::A_BYTES;
            const int ty = t0 + kb * UPD_KB;
            if constexpr (PAIR) {
              // both CTAs' bytes complete the leader's barrier; the leader arms it
              if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * Cf::STAGE_BYTES);
              const uint32_t fb = full0 + 8u * s;
              tma_load_3d_pair(sa, &p.map[3], fb, jb.m0 + rofs, ty, jb.b);             // V[t][d], d contiguous
              tma_load_3d_pair(sa + 64 * UPD_KB * 2, &p.map[3], fb, jb.m0 + rofs + 64, ty, jb.b);
              tma_load_3d_pair(sb, &p.map[4], fb, jb.n0 + rofs, ty, jb.b);             // Z[t][f], f contiguous
              tma_load_3d_pair(sb + 64 * UPD_KB * 2, &p.map[4], fb, jb.n0 + rofs + 64, ty, jb.b);
            } else {
              mbar_arrive_expect_tx(&full[s], Cf::STAGE_BYTES);
              tma_load_3d(sa, &p.map[3], &full[s], jb.m0, ty, jb.b);
              tma_load_3d(sa + 64 * UPD_KB * 2, &p.map[3], &full[s], jb.m0 + 64, ty, jb.b);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                tma_load_3d(sb + q * 64 * UPD_KB * 2, &p.map[4], &full[s], jb.n0 + 64 * q, ty, jb.b);
            }
          }
          jb = jn;
          m = mn;
          have = hn;
        }
        if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
        counters[0] = it;
      }
    } else if (warp == UPD_WARP_MMA) {
      if (lane == 0 && rank == 0) {
        uint32_t it = 0;
        bool ok = true;
        UpdJob jb;
        const uint32_t idesc = idesc_bf16(PAIR ? 256 : 128, 256, true, true);
        bool have = upd_job<PAIR, REV>(p, 0, wk, nwk, jb);
        ChunkMeta m{};
        if (have) m = p.meta[(size_t)jb.b * p.k + jb.chunk];
        for (uint32_t i = 0; ok && have; ++i) {
          UpdJob jn;
          const bool hn = upd_job<PAIR, REV>(p, i + 1, wk, nwk, jn);
          ChunkMeta mn{};
          if (hn) mn = p.meta[(size_t)jn.b * p.k + jn.chunk];   // the next job's, one job ahead
          const int sl = (int)(i & 1);
          const uint32_t u = i >> 1;  // earlier uses of this slot
          const bool got =
              PAIR ? mbar_wait_cluster(&slot_free[sl], (u & 1) ^ 1) : mbar_wait(&slot_free[sl], (u & 1) ^ 1);
          if (!got || *abort_flag) { ok = false; break; }
          tc_fence_after();
          const int t0 = jb.chunk * p.C;
          int kb0, kb1;
          upd_kb_range<REV, UPD_KB>(p, m, t0, kb0, kb1);
          const uint32_t tacc = tmem_base + sl * ACC_COLS;
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(&full[s], ph) || *abort_flag) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(stages + s * Cf::STAGE_BYTES);
            const uint32_t b_addr = a_addr + Cf::A_BYTES;
#pragma unroll
            for (int ks = 0; ks < UPD_KB / 16; ++ks) {
              const uint64_t ad = sdesc_sw128(a_addr + ks * 2048, UPD_KB * 128, 1024);
              const uint64_t bd = sdesc_sw128(b_addr + ks * 2048, UPD_KB * 128, 1024);
              // the chunk's first MMA overwrites the slot: every delta starts from zero
              const uint32_t acc = (kb == kb0 && ks == 0) ? 0u : 1u;
              if constexpr (PAIR) mma_bf16_pair(tacc, ad, bd, idesc, acc);
              else mma_bf16(tacc, ad, bd, idesc, acc);
            }
            if constexpr (PAIR) mma_commit_pair(&empty[s], 3); else mma_commit(&empty[s]);
          }
          if (!ok) break;
          if constexpr (PAIR) mma_commit_pair(&slot_full[sl], 3); else mma_commit(&slot_full[sl]);
          jb = jn;
          m = mn;
          have = hn;
        }
        if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
        counters[1] = it;
        if constexpr (PAIR) mma_commit_pair(drain, 1); else mma_commit(drain);
        mbar_wait(drain, 0);
      }
    }
  }
  __syncthreads();
  // After a timeout: let this CTA's issued but never consumed loads land before
  // the shared memory goes away (each wait is bounded).
  if (*abort_flag && threadIdx.x == 0 && rank == 0) {
    for (uint32_t it = counters[1]; it < counters[0]; ++it)
      mbar_wait(&full[it % STAGES], (it / STAGES) & 1);
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  if (warp == UPD_WARP_MMA) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, 2 * ACC_COLS);
    else tmem_dealloc(tmem_base, 2 * ACC_COLS);
  }
}

// Pairs of CTAs that can be resident at once (a cluster needs two SMs of one
// GPC); 0 when the device cannot run the pair kernel.
template <int KB>
static int max_pairs(cudaStream_t st) {
  static int cached[64];
  static bool have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (have[dev]) return cached[dev];
  int n = 0;
  constexpr int smem = UpdCfg<true, KB>::SMEM;
  if (cudaFuncSetAttribute(upd_kernel<true, KB, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(UPD_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, upd_kernel<true, KB, false, false>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached[dev] = n;
  have[dev] = true;
  return n;
}

static bool pair_update_enabled() {
  const char* e = getenv("IPTTT_UPDATE_CTAS");
  return !(e && e[0] == '1');
}

// The update kernel's register trade (setmaxnreg) balances only at the launch
// register count it was written for; any other count could leave a warpgroup
// waiting for registers, so such a build is refused.
template <bool PAIR, int KB, bool DELTA, bool REV>
static bool upd_regs_ok() {
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, upd_kernel<PAIR, KB, DELTA, REV>) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.numRegs == UPD_REGS_LAUNCH;
}

template <int KB, bool DELTA, bool REV>
static cudaError_t launch_update_kb(const TcParams& p, int num_sms, cudaStream_t st) {
  if (!upd_regs_ok<true, KB, DELTA, REV>() || !upd_regs_ok<false, KB, DELTA, REV>())
    return cudaErrorInvalidDeviceFunction;
  if (p.d % 256 == 0 && pair_update_enabled()) {
    const int np = max_pairs<KB>(st);
    if (np > 0) {
      TcParams q = p;
      q.n_tiles = p.n_tiles / 2;  // 256-row tiles
      constexpr int smem = UpdCfg<true, KB>::SMEM;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * std::max(1, std::min(q.n_tiles, np)), 1, 1);
      cfg.blockDim = dim3(UPD_THREADS, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaFuncSetAttribute(upd_kernel<true, KB, DELTA, REV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess)
        return cudaErrorInvalidValue;
      return cudaLaunchKernelEx(&cfg, upd_kernel<true, KB, DELTA, REV>, q);
    }
  }
  constexpr int smem = UpdCfg<false, KB>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(upd_kernel<false, KB, DELTA, REV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, std::min(p.n_tiles, num_sms));
  upd_kernel<false, KB, DELTA, REV><<<grid, UPD_THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

int update_tokens_per_stage(int C) { return C % 128 == 0 ? 128 : 64; }

cudaError_t launch_update(const TcParams& p, int num_sms, cudaStream_t st) {
  if (p.n_tiles <= 0 || p.dchunks <= 0) return cudaSuccess;
  const int kb = p.upd_kb ? p.upd_kb : update_tokens_per_stage(p.C);
  if (p.rev)
    return kb == 128 ? launch_update_kb<128, false, true>(p, num_sms, st)
                     : launch_update_kb<64, false, true>(p, num_sms, st);
  if (p.delta_out)
    return kb == 128 ? launch_update_kb<128, true, false>(p, num_sms, st)
                     : launch_update_kb<64, true, false>(p, num_sms, st);
  return kb == 128 ? launch_update_kb<128, false, false>(p, num_sms, st)
                   : launch_update_kb<64, false, false>(p, num_sms, st);
}

// ------------------------------------------------------------------ failure-path self test
// One thread waits, with the kernels' bounded wait, on an mbarrier phase that
// nothing completes; when the limit passes it records a timeout in the status word.
__global__ void k_wait_timeout(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, limit_ns)) set_status(status, IPTTT_ERR_TIMEOUT);
  }
}

cudaError_t launch_wait_timeout(int* status, uint64_t limit_ns, cudaStream_t st) {
  k_wait_timeout<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// bf16 tensor [outer][rows][inner] (outer may be 1), box {box_inner, box_rows, 1},
// 128-byte swizzle, zero fill outside the tensor.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                   uint32_t box_inner, uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {inner, rows, outer};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static cudaLaunchConfig_t pair_config(int grid, int smem, cudaStream_t st, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(NTHREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

int pair_gemm_workers(cudaStream_t st) {
  static int cached[64];
  static bool have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (have[dev]) return cached[dev];
  int n = 0;
  constexpr int smem = smem_bytes<FAM_ZV2>();
  if (cudaFuncSetAttribute(tc_kernel<FAM_ZV2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_config(2, smem, st, attr);
    if (cudaOccupancyMaxActiveClusters(&n, tc_kernel<FAM_ZV2>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached[dev] = n;
  have[dev] = true;
  return n;
}

template <int FAM>
static cudaError_t launch(const TcParams& p, int num_sms, cudaStream_t st) {
  constexpr int smem = smem_bytes<FAM>();
  cudaError_t e = cudaFuncSetAttribute(tc_kernel<FAM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if constexpr (is_pair<FAM>()) {
    const int np = pair_gemm_workers(st);
    if (np <= 0) return cudaErrorInvalidConfiguration;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_config(2 * std::max(1, std::min(p.n_tiles, np)), smem, st, attr);
    return cudaLaunchKernelEx(&cfg, tc_kernel<FAM>, p);
  }
  const int grid = std::max(1, std::min(p.n_tiles, num_sms));
  tc_kernel<FAM><<<grid, NTHREADS, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_tc(int fam, const TcParams& p, int num_sms, cudaStream_t st) {
  if (p.n_tiles <= 0) return cudaSuccess;
  switch (fam) {
    case FAM_ZV: return launch<FAM_ZV>(p, num_sms, st);
    case FAM_ZV2: return launch<FAM_ZV2>(p, num_sms, st);
    case FAM_GRAM2: return launch<FAM_GRAM2>(p, num_sms, st);
    case FAM_PZ: return launch<FAM_PZ>(p, num_sms, st);
    case FAM_GRAM: return launch<FAM_GRAM>(p, num_sms, st);
    case FAM_APPLY256: return launch<FAM_APPLY256>(p, num_sms, st);
    default: return launch<FAM_APPLY>(p, num_sms, st);
  }
}

int kind_gateup() { return K_GATEUP; }
int kind_vhat() { return K_VHAT; }
int kind_intra() { return K_INTRA; }

}  // namespace tck
}  // namespace ipttt
