// Token-by-token decoding of the In-Place TTT MLP layer (bf16 path).
//
// A chunk's delta reaches only the chunks after it, and a chunk's outputs come
// from the state before it [iplexlaw.co.kr review of arXiv 2604.06169, §3 and
// §9.1; notes "In-Place Test-Time Training", 方法 › 步骤一/步骤二].  So a token
// decoded inside chunk i needs only the committed state S_i: per token, for every
// row b of the batch,
//   z_t = SiLU(Wgate h_t) * (Wup h_t)                    (rounded to bf16, as Z is)
//   o_t = Wdown0 z_t + m_b (S_i z_t)                       (one fp32 sum, then bf16)
// with m_b = 1 when the token's document began before the chunk.  The chunk's H
// and X0 rows are kept on the device; when the chunk is full, the streaming entry
// point runs on it and commits S_{i+1} exactly as a prefill over the same tokens
// would (target, clip and update need the whole chunk, the conv looks ahead up to
// the chunk end).  The review notes the paper left the decode stage unmeasured
// (§7.5, §8).
//
// The two per-token kernels are batched matrix-vector products bound by HBM: each
// reads Wgate, Wup, Wdown0 once for all rows and every row's bf16 state snapshot.
// From kTensorRows rows on, the gate/up products run as two tcgen05 GEMMs
// (Wgate, Wup as the M operand, the rows' h as an N = 32 operand), whose
// multiply-adds the CUDA cores would otherwise bound.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "aux_kernels.h"
#include "common.cuh"
#include "gemm.h"

namespace ipttt {
namespace {

constexpr int kDecodeMaxRows = 16;  // rows per decode batch
// Rows from which the products run on the tensor cores.  Measured at d=2560, F=9728:
// three rows decode at 35 k tokens/s on the CUDA-core kernels and four at 35 k on
// the tensor cores, where the CUDA-core kernels built for up to 16 rows reach 26 k.
constexpr int kTensorRows = 4;
constexpr int kGemmCols = 32;       // N of those GEMMs: the rows, padded
constexpr int kW0Split = 7;         // K slices of the W0 GEMM (d / 256 pair tiles x 7 fill the SMs)
constexpr int kWarps = 8;           // warps per block

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

// Dot product of the 8 bf16 in one 16-byte word with the 8 bf16 in another, in fp32.
__device__ __forceinline__ float dot8(const uint4 w, const uint4 x) {
  const uint32_t a[4] = {w.x, w.y, w.z, w.w};
  const uint32_t b[4] = {x.x, x.y, x.z, x.w};
  float s = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[e]));
    const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b[e]));
    s = fmaf(fa.x, fb.x, s);
    s = fmaf(fa.y, fb.y, s);
  }
  return s;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Below kTensorRows rows both per-token kernels are persistent: two blocks per SM,
// each warp taking its weight rows in a fixed stride, so the weights stream at
// the full width of the device with no block launched per handful of rows.
// NR: the most rows a build of the kernel takes (kTensorRows - 1).
constexpr int kApplyBatch = 4;   // per operand, in the apply kernel
// 16-byte words of both weight rows a lane requests at once
template <int NR> constexpr int row_words() { return NR <= 3 ? 10 : 6; }

// z[b][f] = bf16(SiLU(Wg[f] . h_b) * (Wu[f] . h_b)) for B <= NR rows.  Each
// warp owns whole rows f (h in shared memory): a lane requests its kRowWords words
// of both weight rows before it uses any, and the warp's sum is taken in a fixed
// order.  Block 0 also files this token's h and x0 rows into the chunk buffers
// (row b at hbuf + b * rs).
template <int NR>
__global__ void __launch_bounds__(kWarps * 32, 2) k_decode_gateup(const __nv_bfloat16* __restrict__ h,
                                                                const __nv_bfloat16* __restrict__ x0,
                                                                const __nv_bfloat16* __restrict__ Wg,
                                                                const __nv_bfloat16* __restrict__ Wu,
                                                                __nv_bfloat16* __restrict__ z, __nv_bfloat16* hbuf,
                                                                __nv_bfloat16* xbuf, long long rs, int B, int d,
                                                                int F) {
  extern __shared__ uint4 hs[];  // [B][d / 8]
  const int dv = d / 8;
  for (int i = threadIdx.x; i < B * dv; i += blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(h)[i];
    hs[i] = v;
    if (blockIdx.x == 0) {
      const int b = i / dv, k = i % dv;
      reinterpret_cast<uint4*>(hbuf + b * rs)[k] = v;
      reinterpret_cast<uint4*>(xbuf + b * rs)[k] = reinterpret_cast<const uint4*>(x0)[i];
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = gridDim.x * kWarps;
  for (int f = blockIdx.x * kWarps + warp; f < F; f += nw) {
    const uint4* wg = reinterpret_cast<const uint4*>(Wg + (size_t)f * d);
    const uint4* wu = reinterpret_cast<const uint4*>(Wu + (size_t)f * d);
    float g[NR], u[NR];
#pragma unroll
    for (int b = 0; b < NR; ++b) g[b] = u[b] = 0.0f;
    for (int k0 = lane; k0 < dv; k0 += 32 * row_words<NR>()) {
      constexpr int RW = row_words<NR>();
      uint4 a[RW], c[RW];
#pragma unroll
      for (int q = 0; q < row_words<NR>(); ++q) {
        const int k = k0 + 32 * q;
        if (k < dv) {
          a[q] = wg[k];
          c[q] = wu[k];
        }
      }
#pragma unroll
      for (int q = 0; q < row_words<NR>(); ++q) {
        const int k = k0 + 32 * q;
        if (k >= dv) break;
#pragma unroll
        for (int b = 0; b < NR; ++b) {
          if (b >= B) break;
          const uint4 x = hs[b * dv + k];
          g[b] += dot8(a[q], x);
          u[b] += dot8(c[q], x);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NR; ++b)
      if (b < B) {
        const float gs = warp_sum(g[b]), us = warp_sum(u[b]);
        if (lane == 0) z[(size_t)b * F + f] = __float2bfloat16_rn(silu_fast(gs) * us);
      }
  }
}

// o[b][j] = bf16(W0[j] . z_b + (m_b ? snap_b[j] . z_b : 0)) for B <= NR rows.
// A block holds two groups of four warps; a group takes one row j at a time, each
// warp a quarter of F, and the quarters are added in a fixed order after a barrier
// of the group's four warps alone.  Per batch of kApplyBatch 16-byte words a lane
// requests the W0 words, then per row b the z_b words (small, L1/L2-resident) and
// the snapshot words before it uses them.
template <int NR>
__global__ void __launch_bounds__(kWarps * 32, 2) k_decode_apply(const __nv_bfloat16* __restrict__ z,
                                                               const __nv_bfloat16* __restrict__ W0,
                                                               const __nv_bfloat16* __restrict__ snap,
                                                               uint32_t mask, __nv_bfloat16* __restrict__ o, int B,
                                                               int d, int F) {
  __shared__ float part[2][kWarps][NR];  // by row parity: a group's next row never overwrites
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp >> 2, quarter = warp & 3;
  const int fv = F / 8;
  const int lo = fv * quarter / 4, hi = fv * (quarter + 1) / 4;
  const int ngrp = gridDim.x * 2;
  int it = 0;
  for (int j = blockIdx.x * 2 + grp; j < d; j += ngrp, ++it) {
    float a0[NR], a1[NR];
#pragma unroll
    for (int b = 0; b < NR; ++b) a0[b] = a1[b] = 0.0f;
    const uint4* w = reinterpret_cast<const uint4*>(W0 + (size_t)j * F);
    for (int k0 = lo + lane; k0 < hi; k0 += 32 * kApplyBatch) {
      uint4 wv[kApplyBatch];
#pragma unroll
      for (int q = 0; q < kApplyBatch; ++q)
        if (k0 + 32 * q < hi) wv[q] = w[k0 + 32 * q];
#pragma unroll
      for (int b = 0; b < NR; ++b) {
        if (b >= B) break;
        const uint4* zb = reinterpret_cast<const uint4*>(z + (size_t)b * F);
        const uint4* sb = reinterpret_cast<const uint4*>(snap + ((size_t)b * d + j) * F);
        const bool cont = (mask >> b) & 1u;
        uint4 zv[kApplyBatch], sv[kApplyBatch];
#pragma unroll
        for (int q = 0; q < kApplyBatch; ++q) {
          const int k = k0 + 32 * q;
          if (k < hi) {
            zv[q] = __ldg(zb + k);
            if (cont) sv[q] = sb[k];
          }
        }
#pragma unroll
        for (int q = 0; q < kApplyBatch; ++q) {
          const int k = k0 + 32 * q;
          if (k >= hi) break;
          a0[b] += dot8(wv[q], zv[q]);
          if (cont) a1[b] += dot8(sv[q], zv[q]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NR; ++b)
      if (b < B) {
        const float s = warp_sum(a0[b]) + warp_sum(a1[b]);
        if (lane == 0) part[it & 1][warp][b] = s;
      }
    // the group's four warps only (barriers 1 and 2; 0 is the block's)
    if (grp == 0) asm volatile("bar.sync 1, 128;" ::: "memory");
    else asm volatile("bar.sync 2, 128;" ::: "memory");
    if (quarter == 0 && lane < B) {
      const float* pp = &part[it & 1][warp][0];
      const float sum = ((pp[lane] + pp[NR + lane]) + pp[2 * NR + lane]) + pp[3 * NR + lane];
      o[(size_t)lane * d + j] = __float2bfloat16_rn(sum);
    }
  }
}

// t[b][j] = m_b ? snap_b[j] . z_b : 0 for many rows b: four warps per (b, j), each a
// quarter of F, summed in a fixed order; each warp streams its own snapshot row, so
// the B copies are read at the full width of the device rather than one W0 row's.
__global__ void __launch_bounds__(kWarps * 32) k_decode_snap(const __nv_bfloat16* __restrict__ z,
                                                           const __nv_bfloat16* __restrict__ snap, uint32_t mask,
                                                           float* __restrict__ t, int B, int d, int F) {
  __shared__ float part[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * (kWarps / 4) + (warp >> 2);  // b d + j
  const int quarter = warp & 3;
  const int b = (int)(r / d), j = (int)(r % d);
  float acc = 0.0f;
  if (b < B && ((mask >> b) & 1u)) {
    const int fv = F / 8;
    const int lo = fv * quarter / 4, hi = fv * (quarter + 1) / 4;
    const uint4* zb = reinterpret_cast<const uint4*>(z + (size_t)b * F);
    const uint4* sb = reinterpret_cast<const uint4*>(snap + ((size_t)b * d + j) * F);
    for (int k0 = lo + lane; k0 < hi; k0 += 32 * kApplyBatch) {
      uint4 zv[kApplyBatch], sv[kApplyBatch];
#pragma unroll
      for (int q = 0; q < kApplyBatch; ++q)
        if (k0 + 32 * q < hi) {
          zv[q] = __ldg(zb + k0 + 32 * q);
          sv[q] = sb[k0 + 32 * q];
        }
#pragma unroll
      for (int q = 0; q < kApplyBatch; ++q)
        if (k0 + 32 * q < hi) acc += dot8(sv[q], zv[q]);
    }
  }
  acc = warp_sum(acc);
  if (lane == 0) part[warp] = acc;
  __syncthreads();
  if (quarter == 0 && lane == 0 && b < B) t[r] = ((part[warp] + part[warp + 1]) + part[warp + 2]) + part[warp + 3];
}

// This token's h and x0 rows into the chunk buffers (row b at hbuf + b * rs).
__global__ void k_decode_file(const __nv_bfloat16* __restrict__ h, const __nv_bfloat16* __restrict__ x0,
                              __nv_bfloat16* hbuf, __nv_bfloat16* xbuf, long long rs, int B, int d) {
  const int dv = d / 8;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B * dv; i += gridDim.x * blockDim.x) {
    const int b = i / dv, k = i % dv;
    reinterpret_cast<uint4*>(hbuf + b * rs)[k] = reinterpret_cast<const uint4*>(h)[i];
    reinterpret_cast<uint4*>(xbuf + b * rs)[k] = reinterpret_cast<const uint4*>(x0)[i];
  }
}

// o[b][j] = bf16(sum over the K slices of part[q][j][b], in slice order, + t[b][j]).
__global__ void k_decode_out(const float* __restrict__ part, const float* __restrict__ t,
                             __nv_bfloat16* __restrict__ o, int B, int d, int slices) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B * d; i += gridDim.x * blockDim.x) {
    const int b = i / d, j = i % d;
    float s = 0.0f;
    for (int q = 0; q < slices; ++q) s += part[((size_t)q * d + j) * kGemmCols + b];
    o[i] = __float2bfloat16_rn(s + t[i]);
  }
}

// z[b][f] = bf16(SiLU(g[f][b]) * u[f][b]) from the GEMMs' fp32 outputs [F][kGemmCols].
__global__ void k_decode_gate_combine(const float* __restrict__ g, const float* __restrict__ u,
                                      __nv_bfloat16* __restrict__ z, int B, int F) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B * F; i += gridDim.x * blockDim.x) {
    const int b = i / F, f = i % F;
    const size_t o = (size_t)f * kGemmCols + b;
    z[i] = __float2bfloat16_rn(silu_fast(g[o]) * u[o]);
  }
}

// Shared memory above the default 48 KB for the gate/up kernel's h rows (B d bf16),
// raised once per device and kernel build to the largest size asked for so far.
template <int NR>
bool decode_smem_ready(int smem) {
  static int granted[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (smem <= granted[dev]) return true;
  if (cudaFuncSetAttribute(k_decode_gateup<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return false;
  granted[dev] = smem;
  return true;
}

// The two per-token kernels on the CUDA cores, built for at most NR rows.
template <int NR>
bool decode_small(const void* h, const void* x0, const void* Wgate, const void* Wup, const void* Wdown0,
                  __nv_bfloat16* z, __nv_bfloat16* hrow, __nv_bfloat16* xrow, const void* snap, uint32_t mask,
                  void* o, long long rs, int B, int d, int F, cudaStream_t st) {
  // the gate/up kernel also files this token's h and x0 rows for the chunk's update
  const int smem = B * d * 2;
  if (smem > 48 * 1024 && !decode_smem_ready<NR>(smem)) return false;
  const int gblocks = std::max(1, std::min(2 * device_sms(), (F + kWarps - 1) / kWarps));
  k_decode_gateup<NR><<<gblocks, kWarps * 32, smem, st>>>(
      static_cast<const __nv_bfloat16*>(h), static_cast<const __nv_bfloat16*>(x0),
      static_cast<const __nv_bfloat16*>(Wgate), static_cast<const __nv_bfloat16*>(Wup), z, hrow, xrow, rs, B, d, F);
  const int ablocks = std::max(1, std::min(2 * device_sms(), (d + 1) / 2));
  k_decode_apply<NR><<<ablocks, kWarps * 32, 0, st>>>(z, static_cast<const __nv_bfloat16*>(Wdown0),
                                                      static_cast<const __nv_bfloat16*>(snap), mask,
                                                      static_cast<__nv_bfloat16*>(o), B, d, F);
  return cudaGetLastError() == cudaSuccess;
}

// Host bookkeeping of a decode state (lives in the caller's host buffer).
struct DecodeHost {
  int32_t B, C, d, F;
  int32_t n;           // tokens of the current chunk already decoded
  int32_t n_starts;    // document starts recorded in the current chunk
  int64_t chunks;      // chunks committed since the reset
  uint32_t cont_mask;  // rows whose current document began before the chunk
  int32_t starts[1];   // [B * C] piece-relative offsets b*C + t of the chunk's starts
};

struct DecodeLayout {
  size_t stream_state, H, X0, Oscr, snap, z, gacc, uacc, tsnap, w0acc, docs, ws, ws_bytes, total;
};

ipttt_params chunk_params(const ipttt_params& p) {
  ipttt_params pc = p;
  pc.T = p.C;
  return pc;
}

bool decode_layout(const ipttt_params& p, DecodeLayout& L) {
  const ipttt_params pc = chunk_params(p);
  const size_t st = ipttt_stream_state_size(&pc), ws = ipttt_workspace_size(&pc);
  if (st == 0 || ws == 0) return false;
  const size_t rows = (size_t)p.B * p.C * p.d * 2;
  size_t off = 0;
  L.stream_state = off; off += al256(st);
  L.H = off;            off += al256(rows);
  L.X0 = off;           off += al256(rows);
  L.Oscr = off;         off += al256(rows);
  L.snap = off;         off += al256((size_t)p.B * p.d * p.F * 2);
  L.z = off;            off += al256((size_t)p.B * p.F * 2);
  L.gacc = off;         off += al256((size_t)p.F * kGemmCols * 4);
  L.uacc = off;         off += al256((size_t)p.F * kGemmCols * 4);
  L.tsnap = off;        off += al256((size_t)p.B * p.d * 4);
  L.w0acc = off;        off += al256((size_t)kW0Split * p.d * kGemmCols * 4);
  L.docs = off;         off += al256((size_t)p.B * p.C * 4);
  L.ws = off;           off += al256(ws);
  L.ws_bytes = ws;
  L.total = off;
  return true;
}

ipttt_status decode_check(const ipttt_params* p) {
  const ipttt_status rc = validate_params(p);
  if (rc != IPTTT_OK) return rc;
  if (p->dtype != IPTTT_BF16 || p->B > kDecodeMaxRows || p->d % 8 != 0 || p->F % 8 != 0)
    return IPTTT_ERR_UNSUPPORTED;
  // the chunk commits go through the streaming path, which takes the per-delta clip only
  if (p->flags & IPTTT_FLAG_STATE_CLIP) return IPTTT_ERR_UNSUPPORTED;
  return IPTTT_OK;
}

size_t host_bytes(const ipttt_params& p) { return sizeof(DecodeHost) + sizeof(int32_t) * (size_t)p.B * p.C; }

}  // namespace
}  // namespace ipttt

using namespace ipttt;

extern "C" {

size_t ipttt_decode_state_size(const ipttt_params* p) {
  if (decode_check(p) != IPTTT_OK) return 0;
  DecodeLayout L;
  return decode_layout(*p, L) ? L.total : 0;
}

size_t ipttt_decode_host_size(const ipttt_params* p) {
  if (decode_check(p) != IPTTT_OK) return 0;
  return host_bytes(*p);
}

ipttt_status ipttt_decode_reset(const ipttt_params* p, void* state, void* host_state, void* stream) {
  const ipttt_status rc = decode_check(p);
  if (rc != IPTTT_OK) return rc;
  if (!state || !host_state) return IPTTT_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(state) % 256 != 0) return IPTTT_ERR_ALIGN;
  DecodeLayout L;
  if (!decode_layout(*p, L)) return IPTTT_ERR_SHAPE;
  uint8_t* base = static_cast<uint8_t*>(state);
  const ipttt_params pc = chunk_params(*p);
  const ipttt_status r2 = ipttt_stream_reset(&pc, base + L.stream_state, stream);
  if (r2 != IPTTT_OK) return r2;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(base + L.snap, 0, (size_t)p->B * p->d * p->F * 2, st) != cudaSuccess) return IPTTT_ERR_CUDA;
  DecodeHost* hs = static_cast<DecodeHost*>(host_state);
  hs->B = p->B;
  hs->C = p->C;
  hs->d = p->d;
  hs->F = p->F;
  hs->n = 0;
  hs->n_starts = 0;
  hs->chunks = 0;
  hs->cont_mask = 0;
  return IPTTT_OK;
}

ipttt_status ipttt_decode_step(const ipttt_params* p, void* state, void* host_state, const void* h, const void* x0,
                               const int32_t* starts_host, const void* Wgate, const void* Wup, const void* Wdown0,
                               const void* conv_w, const void* Wtarget, void* o, void* stream) {
  const ipttt_status rc = decode_check(p);
  if (rc != IPTTT_OK) return rc;
  if (!state || !host_state || !h || !x0 || !Wgate || !Wup || !Wdown0 || !conv_w || !Wtarget || !o)
    return IPTTT_ERR_ARG;
  DecodeHost* hs = static_cast<DecodeHost*>(host_state);
  if (hs->B != p->B || hs->C != p->C || hs->d != p->d || hs->F != p->F) return IPTTT_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(x0) | reinterpret_cast<uintptr_t>(o)) % 16 != 0)
    return IPTTT_ERR_ALIGN;
  DecodeLayout L;
  if (!decode_layout(*p, L)) return IPTTT_ERR_SHAPE;
  uint8_t* base = static_cast<uint8_t*>(state);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int B = p->B, C = p->C, d = p->d, F = p->F;
  const size_t row = (size_t)d * 2;

  // A document start on a row ends its continuation of the previous document.
  if (starts_host)
    for (int b = 0; b < B; ++b)
      if (starts_host[b]) {
        hs->cont_mask &= ~(1u << b);
        hs->starts[hs->n_starts++] = b * C + hs->n;
      }

  __nv_bfloat16* z = reinterpret_cast<__nv_bfloat16*>(base + L.z);
  __nv_bfloat16* hrow = reinterpret_cast<__nv_bfloat16*>(base + L.H + hs->n * row);
  __nv_bfloat16* xrow = reinterpret_cast<__nv_bfloat16*>(base + L.X0 + hs->n * row);
  // (the layout admits only the shapes the forward takes: d and F multiples of 128)
  if (B < kTensorRows) {
    if (!decode_small<kTensorRows - 1>(h, x0, Wgate, Wup, Wdown0, z, hrow, xrow, base + L.snap, hs->cont_mask, o,
                                       (long long)C * d, B, d, F, st))
      return IPTTT_ERR_CUDA;
  } else {
    // g = Wgate h^T and u = Wup h^T as tcgen05 GEMMs (h rows past B read as zeros)
    k_decode_file<<<(B * d / 8 + 255) / 256, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(h),
                                                            static_cast<const __nv_bfloat16*>(x0), hrow, xrow,
                                                            (long long)C * d, B, d);
    gemm::Args g{};
    g.mode = gemm::GM_PLAIN;
    g.M = F;
    g.N = kGemmCols;
    g.K = d;
    g.Bop = {h, (uint64_t)d, (uint64_t)B, 1};
    g.out_kind = gemm::GO_F32;
    g.ldo = kGemmCols;
    g.status = device_status();
    const int sms = device_sms();
    g.A = {Wgate, (uint64_t)d, (uint64_t)F, 1};
    g.out = base + L.gacc;
    if (gemm::run(g, sms, st) != cudaSuccess) return IPTTT_ERR_CUDA;
    g.A = {Wup, (uint64_t)d, (uint64_t)F, 1};
    g.out = base + L.uacc;
    if (gemm::run(g, sms, st) != cudaSuccess) return IPTTT_ERR_CUDA;
    k_decode_gate_combine<<<(B * F + 255) / 256, 256, 0, st>>>(reinterpret_cast<const float*>(base + L.gacc),
                                                               reinterpret_cast<const float*>(base + L.uacc), z, B,
                                                               F);
    // the state copies row by row on their own, then W0 with their products added
    float* tsnap = reinterpret_cast<float*>(base + L.tsnap);
    k_decode_snap<<<(unsigned)(((long long)B * d + kWarps / 4 - 1) / (kWarps / 4)), kWarps * 32, 0, st>>>(
        z, reinterpret_cast<const __nv_bfloat16*>(base + L.snap), hs->cont_mask, tsnap, B, d, F);
    // W0 z_b for all rows as a tcgen05 GEMM (M = d, N = rows padded to 32), K split
    // in kW0Split slices so that the tiles fill the SMs; the slices are added in order
    gemm::Args w0{};
    w0.mode = gemm::GM_PLAIN;
    w0.M = d;
    w0.N = kGemmCols;
    w0.K = F;
    w0.ksplit = F / 128 >= kW0Split ? kW0Split : 1;
    w0.A = {Wdown0, (uint64_t)F, (uint64_t)d, 1};
    w0.Bop = {z, (uint64_t)F, (uint64_t)B, 1};
    w0.out_kind = gemm::GO_F32;
    w0.out = base + L.w0acc;
    w0.ldo = kGemmCols;
    w0.osz = (long long)d * kGemmCols;
    w0.status = device_status();
    if (gemm::run(w0, sms, st) != cudaSuccess) return IPTTT_ERR_CUDA;
    k_decode_out<<<(B * d + 255) / 256, 256, 0, st>>>(reinterpret_cast<const float*>(base + L.w0acc), tsnap,
                                                      static_cast<__nv_bfloat16*>(o), B, d,
                                                      w0.ksplit > 1 ? w0.ksplit : 1);
  }
  if (cudaGetLastError() != cudaSuccess) return IPTTT_ERR_CUDA;

  if (++hs->n < C) return IPTTT_OK;

  // The chunk is complete: commit its update through the streaming entry point (the
  // chunk's outputs it also computes are not needed), then refresh the snapshot.
  std::sort(hs->starts, hs->starts + hs->n_starts);
  int32_t* docs = reinterpret_cast<int32_t*>(base + L.docs);
  if (hs->n_starts > 0 &&
      cudaMemcpyAsync(docs, hs->starts, sizeof(int32_t) * hs->n_starts, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return IPTTT_ERR_CUDA;
  const ipttt_params pc = chunk_params(*p);
  const ipttt_status r2 =
      ipttt_stream_forward(&pc, base + L.stream_state, base + L.H, base + L.X0, Wgate, Wup, Wdown0, conv_w, Wtarget,
                           hs->n_starts > 0 ? docs : nullptr, hs->n_starts, base + L.Oscr, base + L.ws, L.ws_bytes,
                           stream);
  if (r2 != IPTTT_OK) return r2;
  const Shape s{B, C, d, F, C, 1};
  if (aux::state_snapshot(reinterpret_cast<const float*>(base + L.stream_state), base + L.snap, s, st) !=
      cudaSuccess)
    return IPTTT_ERR_CUDA;
  hs->n = 0;
  hs->n_starts = 0;
  hs->chunks += 1;
  hs->cont_mask = (B >= 32) ? 0xffffffffu : ((1u << B) - 1u);  // every row continues into the next chunk
  return IPTTT_OK;
}

ipttt_status ipttt_decode_export(const ipttt_params* p, const void* state, float* S_out, void* stream) {
  const ipttt_status rc = decode_check(p);
  if (rc != IPTTT_OK) return rc;
  if (!state || !S_out) return IPTTT_ERR_ARG;
  DecodeLayout L;
  if (!decode_layout(*p, L)) return IPTTT_ERR_SHAPE;
  const ipttt_params pc = chunk_params(*p);
  return ipttt_stream_export(&pc, static_cast<const uint8_t*>(state) + L.stream_state, S_out, stream);
}

}  // extern "C"
