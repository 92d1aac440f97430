// A general bf16 tensor-core GEMM (tcgen05, fp32 accumulators in TMEM) for the
// backward of the layer, whose products come in three shapes:
//
//   GM_PLAIN       out[m][n]            = s * sum_k A(m, k) B(k, n)
//                  (with ksplit > 1: out[q][m][n] over the q-th of ksplit slices of K,
//                  for a caller that adds them in a fixed order)
//   GM_CHUNK_ROWS  out[b][t0 + m][n]   (=, +=) s[b][i] * sum_k A(b, t0 + m, k) B_i(k, n)
//                  for the tokens t0 + m of chunk i (rows outside the chosen
//                  document segment of the chunk are left alone), B_i taken from
//                  chunk i's slot of a stack of [d][F] matrices
//   GM_CHUNK_K     out[i][b][m][n]      = sum over the tokens t of chunk i of A(b, t, m) B(b, t, n)
//
// Operands are bf16 arrays {outer, rows, inner} read through 128-byte-swizzled
// TMA boxes, in one of two orders: K-major (k is the inner, contiguous index) or
// MN-major (m, resp. n, is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"

namespace ipttt {
namespace gemm {

enum Mode { GM_PLAIN = 0, GM_CHUNK_ROWS = 1, GM_CHUNK_K = 2 };
// Rows of a chunk an GM_CHUNK_ROWS output keeps: all, the chunk's last document
// segment, or its first segment when it continues the previous chunk's document.
enum Rows { GR_ALL = 0, GR_LAST = 1, GR_FIRST = 2 };
enum Out { GO_F32 = 0, GO_F32_ADD = 1, GO_BF16 = 2 };

// A bf16 operand: a row-major {outer, rows, inner} array (inner contiguous).
struct Operand {
  const void* base;
  uint64_t inner, rows, outer;
};

struct Args {
  Operand A, Bop;        // the tensor maps are made by run() for the form it picks
  int a_mn, b_mn;        // operand order (1: MN-major); the per-chunk-K form takes both MN-major
  int mode;              // Mode
  int M, N, K;           // PLAIN: all three; CHUNK_ROWS: N, K; CHUNK_K: M, N
  int B, T, C, k;        // chunk modes: rows, tokens per row, chunk length, chunks per row
  int chunk0, nchunks;   // chunk modes: chunks [chunk0, chunk0 + nchunks) of every row
  int nslots;            // CHUNK_ROWS: B_i lies in slot i % nslots (outer index slot * B + b)
  int out_kind;          // Out
  void* out;             // fp32 or bf16, rows of ldo elements
  long long ldo;         // elements between output rows
  long long osz;         // elements between output matrices (per b, or per slot * B + b)
  const float* scale;    // optional [B][k] scale (chunk modes) or [1] (PLAIN)
  const ChunkMeta* meta; // CHUNK_ROWS with rows != GR_ALL: [B][k]
  int rows;              // Rows
  int ksplit;            // PLAIN: K in this many slices (0 or 1: one), slice s written at out + s * osz
  int* status;           // device status word (timeouts)
  int chunk_base;        // CHUNK_K: chunk i's matrices go to index i - chunk_base of out
};

// Launches the persistent kernel: on clusters of two CTAs (256-row tiles) when the
// rows are at least 256 (and, per chunk rows, the chunk a multiple of 256), else
// on up to num_sms single CTAs.  cudaErrorInvalidValue when N is not a multiple
// of 32, a size is not positive or a tensor map cannot be made.
cudaError_t run(const Args& a, int num_sms, cudaStream_t st);

}  // namespace gemm
}  // namespace ipttt
