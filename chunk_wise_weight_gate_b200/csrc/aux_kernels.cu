// Non-tensor-core kernels of libipttt: document/chunk metadata, the masked
// depthwise conv of the LM-aligned target, the clip factor, state layout
// conversions, and the all-fp32 (SIMT) path.
//
// Sources: cloud.tencent.com "榨干MLP的剩余价值", 详细步骤 3 (depthwise conv of
// kernel 5 over the token embeddings, no look past the chunk) and 4 (Frobenius
// clip); iplexlaw.co.kr review of arXiv 2604.06169, §6 (chunk and document
// boundaries, fast weight reset per document); lijianxiong.blog notes
// "In-Place Test-Time Training", 方法 (gated MLP, apply/update, Hebbian rule).
#include <cuda_bf16.h>
#include <math.h>

#include "aux_kernels.h"
#include "common.cuh"

namespace ipttt {
namespace aux {

constexpr int kTaps = 5;

// ------------------------------------------------------------------ metadata
__global__ void k_fill_u8(uint8_t* p, size_t n, uint8_t v) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    p[i] = v;
}

// flags[b*T + t] = 1 at every document start.  A row start is a start unless the
// row continues a document from an earlier streaming piece (row_cont[b] != 0).
__global__ void k_mark_starts(uint8_t* flags, int B, int T, const int32_t* ds, int n, const int32_t* row_cont,
                              int* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const long long g = ds[i];
    if (g < 0 || g >= (long long)B * T || (i > 0 && (long long)ds[i - 1] >= g))
      set_status(status, IPTTT_ERR_ARG);
    else
      flags[g] = 1;
  }
  if (i < B && (row_cont == nullptr || row_cont[i] == 0)) flags[(size_t)i * T] = 1;
}

// One block per (row, chunk): the chunk's flags are scanned by all threads and
// reduced to the first start after the chunk start, the last start, and "any".
__global__ void k_chunk_meta(const uint8_t* flags, ChunkMeta* meta, int B, int T, int C, int k) {
  __shared__ int s_first, s_last, s_any;
  const int i = blockIdx.x;
  const int b = i / k, c = i % k;
  const int s = c * C, e = min(s + C, T);
  const uint8_t* f = flags + (size_t)b * T;
  if (threadIdx.x == 0) {
    s_first = e;
    s_last = -1;
    s_any = 0;
  }
  __syncthreads();
  int first = e, last = -1;
  for (int t = s + threadIdx.x; t < e; t += blockDim.x) {
    if (f[t]) {
      if (t > s) first = min(first, t);
      last = max(last, t);
    }
  }
  if (first < e) atomicMin(&s_first, first);
  if (last >= 0) {
    atomicMax(&s_last, last);
    s_any = 1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    ChunkMeta m;
    m.first_end = s_first;
    m.last_start = s_last >= 0 ? s_last : s;
    m.cont = f[s] ? 0 : 1;
    m.has_start = s_any;
    meta[i] = m;
  }
}

cudaError_t build_meta(uint8_t* flags, ChunkMeta* meta, const Shape& s, const int32_t* doc_starts, int n_doc,
                       const int32_t* row_cont, int* status, cudaStream_t st) {
  const size_t n = (size_t)s.B * s.T;
  k_fill_u8<<<(unsigned)std::min<size_t>((n + 255) / 256, 4096), 256, 0, st>>>(flags, n, 0);
  const int nt = std::max(n_doc, s.B);
  k_mark_starts<<<(nt + 255) / 256, 256, 0, st>>>(flags, s.B, s.T, doc_starts, n_doc, row_cont, status);
  k_chunk_meta<<<s.B * s.k, 256, 0, st>>>(flags, meta, s.B, s.T, s.C, s.k);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ conv
// U[b,t,c] = sum_o conv_w[c,o] X0[b,t+o,c]; tap o is dropped (and every later
// one) once t+o reaches the chunk end or T, or a document starts at t+o.
// A thread owns VEC channels of one row over RUN consecutive tokens: it keeps
// its 5 x VEC taps and a 5-row window of X0 in registers, so every X0 element
// is read about once and a warp's loads and stores cover contiguous bytes.
constexpr int kConvRun = 16;

template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T* p, float (&out)[VEC]) {
#pragma unroll
  for (int v = 0; v < VEC; ++v) out[v] = to_f<T>(p[v]);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&out)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
    out[2 * e] = __low2float(h);
    out[2 * e + 1] = __high2float(h);
  }
}
template <>
__device__ __forceinline__ void load_vec<float, 4>(const float* p, float (&out)[4]) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  out[0] = q.x; out[1] = q.y; out[2] = q.z; out[3] = q.w;
}
template <typename T, int VEC>
__device__ __forceinline__ void store_vec(T* p, const float (&in)[VEC]) {
#pragma unroll
  for (int v = 0; v < VEC; ++v) p[v] = from_f<T>(in[v]);
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 8>(__nv_bfloat16* p, const float (&in)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 h = __floats2bfloat162_rn(in[2 * e], in[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ void store_vec<float, 4>(float* p, const float (&in)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
}

template <typename T, int VEC>
__global__ void __launch_bounds__(256) k_conv(const T* __restrict__ X0, const T* __restrict__ cw,
                                              const uint8_t* __restrict__ flags, T* __restrict__ U, int B, int Tn,
                                              int d, int C) {
  const int groups = d / VEC;
  const int runs = (Tn + kConvRun - 1) / kConvRun;
  const size_t total = (size_t)B * runs * groups;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int g = (int)(idx % groups);
    const size_t rr = idx / groups;
    const int run = (int)(rr % runs);
    const int b = (int)(rr / runs);
    float w[kTaps][VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v)
#pragma unroll
      for (int o = 0; o < kTaps; ++o) w[o][v] = to_f<T>(cw[(size_t)(g * VEC + v) * kTaps + o]);
    const int t_begin = run * kConvRun;
    const int t_end = min(t_begin + kConvRun, Tn);
    const uint8_t* f = flags + (size_t)b * Tn;
    const T* xb = X0 + (size_t)b * Tn * d + (size_t)g * VEC;
    T* ub = U + (size_t)b * Tn * d + (size_t)g * VEC;
    float win[kTaps][VEC];
#pragma unroll
    for (int o = 0; o < kTaps - 1; ++o) {
      const int src = t_begin + o;
#pragma unroll
      for (int v = 0; v < VEC; ++v) win[o + 1][v] = 0.0f;
      if (src < Tn) load_vec<T, VEC>(xb + (size_t)src * d, win[o + 1]);
    }
    for (int t = t_begin; t < t_end; ++t) {
      // slide: win[o] holds X0[t + o]
#pragma unroll
      for (int o = 0; o < kTaps - 1; ++o)
#pragma unroll
        for (int v = 0; v < VEC; ++v) win[o][v] = win[o + 1][v];
      const int nxt = t + kTaps - 1;
#pragma unroll
      for (int v = 0; v < VEC; ++v) win[kTaps - 1][v] = 0.0f;
      if (nxt < Tn) load_vec<T, VEC>(xb + (size_t)nxt * d, win[kTaps - 1]);
      const int cend = min((t / C + 1) * C, Tn);
      int ntaps = 1;
#pragma unroll
      for (int o = 1; o < kTaps; ++o)
        if (ntaps == o && t + o < cend && !f[t + o]) ntaps = o + 1;
      float acc[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = 0.0f;
#pragma unroll
      for (int o = 0; o < kTaps; ++o)
        if (o < ntaps) {
#pragma unroll
          for (int v = 0; v < VEC; ++v) acc[v] = fmaf(w[o][v], win[o][v], acc[v]);
        }
      store_vec<T, VEC>(ub + (size_t)t * d, acc);
    }
  }
}

// bf16 masked depthwise conv: each thread 8 channels x kRun16 rows, its whole
// (rows + 4)-row window requested at once so that every thread keeps 12 loads in
// flight, two blocks of 256 threads per SM (the generic kernel above slides one
// row at a time and waits on each);
// two channels per FMA (fma.rn.f32x2), taps in order from zero, one bf16 rounding:
// the generic kernel's arithmetic, bit for bit.
constexpr int kRun16 = 8;

__device__ __forceinline__ unsigned long long cv_f2pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ unsigned long long cv_fma2(unsigned long long a, unsigned long long b,
                                                      unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__global__ void __launch_bounds__(256, 2) k_conv_bf16(const __nv_bfloat16* __restrict__ X0,
                                                   const __nv_bfloat16* __restrict__ cw,
                                                   const uint8_t* __restrict__ flags, __nv_bfloat16* __restrict__ U,
                                                   int B, int Tn, int d, int C) {
  const int groups = d / 8;
  const int runs = (Tn + kRun16 - 1) / kRun16;
  const size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (idx >= (size_t)B * runs * groups) return;
  const int g = (int)(idx % groups);
  const size_t rr = idx / groups;
  const int run = (int)(rr % runs);
  const int b = (int)(rr / runs);
  const int t0 = run * kRun16;
  const __nv_bfloat16* xb = X0 + ((size_t)b * Tn + t0) * d + (size_t)g * 8;
  uint4 x[kRun16 + 4];
#pragma unroll
  for (int q = 0; q < kRun16 + 4; ++q)
    x[q] = (t0 + q < Tn) ? __ldg(reinterpret_cast<const uint4*>(xb + (size_t)q * d)) : make_uint4(0u, 0u, 0u, 0u);
  // taps: channel pairs (2p, 2p+1) of tap o as one fp32 pair
  uint4 wr[5];
  const uint4* wsrc = reinterpret_cast<const uint4*>(cw + (size_t)g * 8 * kTaps);
#pragma unroll
  for (int q = 0; q < 5; ++q) wr[q] = __ldg(wsrc + q);
  const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(wr);
  unsigned long long wp[kTaps][4];
#pragma unroll
  for (int o = 0; o < kTaps; ++o)
#pragma unroll
    for (int p = 0; p < 4; ++p)
      wp[o][p] = cv_f2pack(__bfloat162float(wb[(2 * p) * kTaps + o]), __bfloat162float(wb[(2 * p + 1) * kTaps + o]));
  // start flags of rows t0 + 1 .. t0 + kRun16 + 3 (a tap past one of them is dropped)
  const uint8_t* f = flags + (size_t)b * Tn;
  uint32_t st = 0;
#pragma unroll
  for (int q = 1; q < kRun16 + 4; ++q)
    if (t0 + q < Tn && f[t0 + q]) st |= 1u << q;
  __nv_bfloat16* ub = U + ((size_t)b * Tn + t0) * d + (size_t)g * 8;
#pragma unroll
  for (int r = 0; r < kRun16; ++r) {
    const int t = t0 + r;
    if (t >= Tn) break;
    const int cend = min((t / C + 1) * C, Tn);
    int n = 1;
#pragma unroll
    for (int o = 1; o < kTaps; ++o)
      if (n == o && t + o < cend && !((st >> (r + o)) & 1u)) n = o + 1;
    unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int o = 0; o < kTaps; ++o) {
      if (o < n) {
        const uint32_t xw[4] = {x[r + o].x, x[r + o].y, x[r + o].z, x[r + o].w};
#pragma unroll
        for (int p = 0; p < 4; ++p)
          acc[p] = cv_fma2(wp[o][p], cv_f2pack(__uint_as_float(xw[p] << 16), __uint_as_float(xw[p] & 0xffff0000u)),
                           acc[p]);
      }
    }
    uint32_t ow[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float lo, hi;
      asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc[p]));
      __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
      ow[p] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(ub + (size_t)r * d) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
}

cudaError_t conv_target(int dtype, const void* X0, const void* cw, const uint8_t* flags, void* U, const Shape& s,
                        cudaStream_t st) {
  const int blocks = 148 * 8;
  if (dtype == IPTTT_BF16 && s.d % 8 == 0) {
    const size_t threads = (size_t)s.B * ((s.T + kRun16 - 1) / kRun16) * (s.d / 8);
    k_conv_bf16<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>((const __nv_bfloat16*)X0,
                                                                  (const __nv_bfloat16*)cw, flags,
                                                                  (__nv_bfloat16*)U, s.B, s.T, s.d, s.C);
  } else if (dtype == IPTTT_BF16)
    k_conv<__nv_bfloat16, 1><<<blocks, 256, 0, st>>>((const __nv_bfloat16*)X0, (const __nv_bfloat16*)cw, flags,
                                                       (__nv_bfloat16*)U, s.B, s.T, s.d, s.C);
  else if (s.d % 4 == 0)
    k_conv<float, 4><<<blocks, 256, 0, st>>>((const float*)X0, (const float*)cw, flags, (float*)U, s.B, s.T, s.d,
                                             s.C);
  else
    k_conv<float, 1><<<blocks, 256, 0, st>>>((const float*)X0, (const float*)cw, flags, (float*)U, s.B, s.T, s.d,
                                             s.C);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ clip factor
__device__ __forceinline__ float clip_alpha(double sumsq, float eta, float tau) {
  const float nrm = eta * (float)sqrt(fmax(sumsq, 0.0));
  return (tau > 0.0f && isfinite(tau) && nrm > tau) ? tau / nrm : 1.0f;
}

// alpha[i] from the per-tile-pair Gram partials of ||V^T Z||_F^2, summed in a
// fixed order.
__global__ void k_alpha_from_partials(const float* partials, float* alpha, int n, int npairs, float eta,
                                      float tau) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  double s = 0.0;
  for (int q = 0; q < npairs; ++q) s += (double)partials[(size_t)i * npairs + q];
  alpha[i] = clip_alpha(s, eta, tau);
}

cudaError_t alpha_from_partials(const float* partials, float* alpha, int n, int npairs, float eta, float tau,
                                cudaStream_t st) {
  k_alpha_from_partials<<<(n + 127) / 128, 128, 0, st>>>(partials, alpha, n, npairs, eta, tau);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ state layouts
// The bf16 path keeps S [d][F] (fp32) as 128 x 128 tiles, tile (mt, nt) at
// ((mt * F/128) + nt) * 16384, element (r, c) of a tile at ((c/4) * 128 + r) * 4 + c%4,
// so a tile is one contiguous 64 KB block laid out as the TMEM lanes read it.
__device__ __forceinline__ size_t blocked_index(int r, int c, int F) {
  const size_t tile = (size_t)(r >> 7) * (F >> 7) + (c >> 7);
  return tile * 16384 + ((size_t)((c & 127) >> 2) * 128 + (r & 127)) * 4 + (c & 3);
}

__global__ void k_blocked_to_rowmajor(const float* Sb, float* out, int B, int d, int F) {
  const size_t total = (size_t)B * d * F;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % F);
    const size_t br = i / F;
    const int r = (int)(br % d);
    const size_t b = br / d;
    out[i] = Sb[b * d * F + blocked_index(r, c, F)];
  }
}

__global__ void k_blocked_to_bf16(const float* Sb, __nv_bfloat16* out, int B, int d, int F) {
  const size_t total = (size_t)B * d * F;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % F);
    const size_t br = i / F;
    const int r = (int)(br % d);
    const size_t b = br / d;
    out[i] = __float2bfloat16_rn(Sb[b * d * F + blocked_index(r, c, F)]);
  }
}

// Four consecutive columns (c % 4 == 0) stay consecutive in the blocked layout, so
// each thread moves one float4 (F % 128 == 0).
__global__ void k_rowmajor_to_blocked(const float* in, float* Sb, int B, int d, int F) {
  const size_t total4 = (size_t)B * d * F / 4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total4; i += (size_t)gridDim.x * blockDim.x) {
    const size_t e = 4 * i;
    const int c = (int)(e % F);
    const size_t br = e / F;
    const int r = (int)(br % d);
    const size_t b = br / d;
    *reinterpret_cast<float4*>(Sb + b * d * F + blocked_index(r, c, F)) = reinterpret_cast<const float4*>(in)[i];
  }
}

cudaError_t state_import_blocked(const float* in, float* Sb, const Shape& s, cudaStream_t st) {
  if (!in) return cudaMemsetAsync(Sb, 0, (size_t)s.B * s.d * s.F * sizeof(float), st);
  k_rowmajor_to_blocked<<<148 * 8, 256, 0, st>>>(in, Sb, s.B, s.d, s.F);
  return cudaGetLastError();
}

cudaError_t state_export(bool blocked, const float* S, float* out, const Shape& s, cudaStream_t st) {
  const size_t n = (size_t)s.B * s.d * s.F;
  if (!blocked) return cudaMemcpyAsync(out, S, n * sizeof(float), cudaMemcpyDeviceToDevice, st);
  k_blocked_to_rowmajor<<<148 * 8, 256, 0, st>>>(S, out, s.B, s.d, s.F);
  return cudaGetLastError();
}

cudaError_t state_snapshot(const float* Sb, void* snap_bf16, const Shape& s, cudaStream_t st) {
  k_blocked_to_bf16<<<148 * 8, 256, 0, st>>>(Sb, (__nv_bfloat16*)snap_bf16, s.B, s.d, s.F);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ fp32 SIMT path
// C(m,n) = sum_k A(m,k) B(n,k) with arbitrary element strides, 64 x 64 tiles,
// 16 x 16 threads of 4 x 4 outputs, and up to two B operands sharing A.
constexpr int ST = 64, SK = 16;

__global__ void __launch_bounds__(256) k_simt_gemm(SimtArgs a) {
  __shared__ float As[SK][ST + 1];
  __shared__ float Bs0[SK][ST + 1];
  __shared__ float Bs1[SK][ST + 1];
  const int b = blockIdx.z;
  const int m0 = blockIdx.y * ST, n0 = blockIdx.x * ST;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const float* A = a.A + b * a.sab;
  const float* B0 = a.B0 + b * a.s0b;
  const float* B1 = a.B1 ? a.B1 + b * a.s1b : nullptr;
  float acc0[4][4] = {}, acc1[4][4] = {};
  for (int k0 = 0; k0 < a.K; k0 += SK) {
    for (int e = threadIdx.x; e < ST * SK; e += 256) {
      const int mm = e / SK, kk = e % SK;
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < a.M && gk < a.K) ? A[gm * a.sam + gk * a.sak] : 0.0f;
      const int gn = n0 + mm;
      Bs0[kk][mm] = (gn < a.N && gk < a.K) ? B0[gn * a.s0n + gk * a.s0k] : 0.0f;
      if (B1) Bs1[kk][mm] = (gn < a.N && gk < a.K) ? B1[gn * a.s1n + gk * a.s1k] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float av[4], bv0[4], bv1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        bv0[i] = Bs0[kk][tx * 4 + i];
        bv1[i] = B1 ? Bs1[kk][tx * 4 + i] : 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          acc0[i][jj] = fmaf(av[i], bv0[jj], acc0[i][jj]);
          acc1[i][jj] = fmaf(av[i], bv1[jj], acc1[i][jj]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
    const int t = a.row0 + m;  // token index for the token-row modes
    bool keep_row = true;
    if (a.mode == SM_V || a.mode == SM_ACC_L) {
      const int c = t / a.C;
      keep_row = t >= a.meta[(size_t)b * a.k + c].last_start;
    } else if (a.mode == SM_APPLY) {
      const ChunkMeta cm = a.meta[(size_t)b * a.k + a.chunk];
      keep_row = cm.cont && t < cm.first_end;
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int n = n0 + tx * 4 + jj;
      if (n >= a.N) continue;
      float* o = a.out + b * a.sob + (long long)m * a.som + (long long)n * a.son;
      switch (a.mode) {
        case SM_Z: *o = silu_precise(acc0[i][jj]) * acc1[i][jj]; break;
        case SM_V: *o = keep_row ? acc0[i][jj] : 0.0f; break;
        case SM_RAW: *o = acc0[i][jj]; break;
        case SM_ACC: *o += acc0[i][jj]; break;
        case SM_ACC_L:
          if (keep_row) *o += acc0[i][jj];
          break;
        case SM_APPLY: {
          const float dv = keep_row ? acc1[i][jj] : 0.0f;
          *o = acc0[i][jj] + dv +
               (a.resid ? a.resid[b * a.sob + (long long)m * a.som + (long long)n * a.son] : 0.0f);
          if (a.out2) a.out2[b * a.sob + (long long)m * a.som + (long long)n * a.son] = dv;
        } break;
      }
    }
  }
}

cudaError_t simt_gemm(const SimtArgs& a, int batches, cudaStream_t st) {
  dim3 grid((a.N + ST - 1) / ST, (a.M + ST - 1) / ST, batches);
  k_simt_gemm<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

// Sum of squares of each row-b slice [n] of x, as per-block partials [B][nblk].
__global__ void k_sumsq_partials(const float* x, size_t n, double* part, int nblk) {
  __shared__ double sh[256];
  const int b = blockIdx.y;
  const float* xb = x + b * n;
  double s = 0.0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)nblk * blockDim.x)
    s += (double)xb[i] * (double)xb[i];
  sh[threadIdx.x] = s;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[(size_t)b * nblk + blockIdx.x] = sh[0];
}

__global__ void k_alpha_direct(const double* part, int nblk, float* alpha, int B, int k, int chunk, float eta,
                               float tau) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  double s = 0.0;
  for (int q = 0; q < nblk; ++q) s += part[(size_t)b * nblk + q];
  alpha[(size_t)b * k + chunk] = clip_alpha(s, eta, tau);
}

// S = (chunk holds a document start ? 0 : S) + alpha * eta * raw, per row b.
__global__ void k_state_update(float* S, const float* raw, size_t n, const float* alpha, const ChunkMeta* meta,
                               int k, int chunk, float eta) {
  const int b = blockIdx.y;
  const float ae = alpha[(size_t)b * k + chunk] * eta;
  const bool keep = !meta[(size_t)b * k + chunk].has_start;
  float* Sb = S + b * n;
  const float* rb = raw + b * n;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    Sb[i] = fmaf(ae, rb[i], keep ? Sb[i] : 0.0f);
}

// The clip on the accumulated state (an ablation): per row b,
//   S = c (keep S + eta raw),  c = tau / ||keep S + eta raw||_F when that norm exceeds tau, else 1,
// with c stored in alpha[b][chunk].
__global__ void k_state_accum(float* S, const float* raw, size_t n, const ChunkMeta* meta, int k, int chunk,
                              float eta) {
  const int b = blockIdx.y;
  const bool keep = !meta[(size_t)b * k + chunk].has_start;
  float* Sb = S + b * n;
  const float* rb = raw + b * n;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    Sb[i] = fmaf(eta, rb[i], keep ? Sb[i] : 0.0f);
}

__global__ void k_state_scale(float* S, size_t n, const float* alpha, int k, int chunk) {
  const int b = blockIdx.y;
  const float c = alpha[(size_t)b * k + chunk];
  if (c == 1.0f) return;
  float* Sb = S + b * n;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    Sb[i] *= c;
}

cudaError_t simt_update_state_clipped(float* S, const float* raw, double* part, float* alpha, const ChunkMeta* meta,
                                      const Shape& s, int chunk, float eta, float tau, cudaStream_t st) {
  const size_t n = (size_t)s.d * s.F;
  const int nblk = 64;
  k_state_accum<<<dim3(256, s.B), 256, 0, st>>>(S, raw, n, meta, s.k, chunk, eta);
  k_sumsq_partials<<<dim3(nblk, s.B), 256, 0, st>>>(S, n, part, nblk);
  k_alpha_direct<<<(s.B + 63) / 64, 64, 0, st>>>(part, nblk, alpha, s.B, s.k, chunk, 1.0f, tau);
  k_state_scale<<<dim3(256, s.B), 256, 0, st>>>(S, n, alpha, s.k, chunk);
  return cudaGetLastError();
}

// The accumulated-state clip on the bf16 path, for states of d F = tens of millions
// of values: one pass forms keep S + eta raw and its partial sums of squares (four
// values per thread and step, fixed-order block sums), a second scales the state
// by c and writes its bf16 copy for the apply.
constexpr int kClipBlocks = 148 * 4;

__global__ void __launch_bounds__(256) k_state_accum_sumsq(float* S, const float* raw, size_t n4,
                                                           const ChunkMeta* meta, int k, int chunk, float eta,
                                                           double* part) {
  __shared__ double sh[256];
  const int b = blockIdx.y;
  const bool keep = !meta[(size_t)b * k + chunk].has_start;
  float4* Sb = reinterpret_cast<float4*>(S) + b * n4;
  const float4* rb = reinterpret_cast<const float4*>(raw) + b * n4;
  double acc = 0.0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    const float4 r = rb[i];
    float4 v = keep ? Sb[i] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    v.x = fmaf(eta, r.x, v.x);
    v.y = fmaf(eta, r.y, v.y);
    v.z = fmaf(eta, r.z, v.z);
    v.w = fmaf(eta, r.w, v.w);
    Sb[i] = v;
    acc += ((double)v.x * v.x + (double)v.y * v.y) + ((double)v.z * v.z + (double)v.w * v.w);
  }
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[(size_t)b * gridDim.x + blockIdx.x] = sh[0];
}

__global__ void __launch_bounds__(256) k_state_scale_copy(float* S, __nv_bfloat16* snap, size_t n4,
                                                          const float* alpha, int k, int chunk) {
  const int b = blockIdx.y;
  const float c = alpha[(size_t)b * k + chunk];
  float4* Sb = reinterpret_cast<float4*>(S) + b * n4;
  uint2* out = snap ? reinterpret_cast<uint2*>(snap) + b * n4 : nullptr;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    float4 v = Sb[i];
    if (c != 1.0f) {
      v.x *= c;
      v.y *= c;
      v.z *= c;
      v.w *= c;
      Sb[i] = v;
    }
    if (out) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
      out[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
  }
}

cudaError_t state_clip_step(float* S, const float* raw, double* part, float* alpha, const ChunkMeta* meta,
                            const Shape& s, int chunk, float eta, float tau, void* snap_bf16, cudaStream_t st) {
  const size_t n = (size_t)s.d * s.F;
  if (n % 4 != 0) return cudaErrorInvalidValue;
  k_state_accum_sumsq<<<dim3(kClipBlocks, s.B), 256, 0, st>>>(S, raw, n / 4, meta, s.k, chunk, eta, part);
  k_alpha_direct<<<(s.B + 63) / 64, 64, 0, st>>>(part, kClipBlocks, alpha, s.B, s.k, chunk, 1.0f, tau);
  k_state_scale_copy<<<dim3(kClipBlocks, s.B), 256, 0, st>>>(S, static_cast<__nv_bfloat16*>(snap_bf16), n / 4,
                                                               alpha, s.k, chunk);
  return cudaGetLastError();
}

cudaError_t simt_update_state(float* S, const float* raw, double* part, float* alpha, const ChunkMeta* meta,
                              const Shape& s, int chunk, float eta, float tau, cudaStream_t st) {
  const size_t n = (size_t)s.d * s.F;
  const int nblk = 64;
  k_sumsq_partials<<<dim3(nblk, s.B), 256, 0, st>>>(raw, n, part, nblk);
  k_alpha_direct<<<(s.B + 63) / 64, 64, 0, st>>>(part, nblk, alpha, s.B, s.k, chunk, eta, tau);
  k_state_update<<<dim3(256, s.B), 256, 0, st>>>(S, raw, n, alpha, meta, s.k, chunk, eta);
  return cudaGetLastError();
}

}  // namespace aux
}  // namespace ipttt

namespace ipttt {
namespace aux {

// out[b,t,:] = in[b,t,:] on rows inside their chunk's last document segment, 0 elsewhere.
template <typename T>
__global__ void k_mask_last_segment(const T* in, T* out, const ChunkMeta* meta, int B, int Tn, int d, int C, int k) {
  const size_t total = (size_t)B * Tn * d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const size_t bt = i / d;
    const int t = (int)(bt % Tn);
    const int b = (int)(bt / Tn);
    const bool keep = t >= meta[(size_t)b * k + t / C].last_start;
    out[i] = keep ? in[i] : from_f<T>(0.0f);
  }
}

cudaError_t mask_last_segment(int dtype, const void* in, void* out, const ChunkMeta* meta, const Shape& s,
                              cudaStream_t st) {
  if (dtype == IPTTT_BF16)
    k_mask_last_segment<__nv_bfloat16><<<148 * 8, 256, 0, st>>>((const __nv_bfloat16*)in, (__nv_bfloat16*)out, meta,
                                                                 s.B, s.T, s.d, s.C, s.k);
  else
    k_mask_last_segment<float><<<148 * 8, 256, 0, st>>>((const float*)in, (float*)out, meta, s.B, s.T, s.d, s.C, s.k);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ context parallelism
// One block per (row b, 128 x 128 state tile, quarter of 32 tile rows).  With plan
// = [row_cont | first_rank | prefix_chunks | keep] (each [B]):
//   S_in      = sum over ranks j in [first_rank[b], rank) of gathered[j][b]
//   snapshot S_i (ring slot i, bf16, row-major) += S_in   for chunks i < prefix_chunks[b]
//   S_final   = gathered[rank][b] + (keep[b] ? S_in : 0)   (row-major fp32, optional)
// The aggregates are in the state's blocked order, where the 32 rows of a quarter
// and 4 columns form one 512-byte run, so the reads are whole runs; the rows go
// through shared memory (rows padded to 33 float4) to the row-major writes.  The
// sum runs in rank order, the same on every rank.
__global__ void __launch_bounds__(256) k_cp_combine(const float* __restrict__ gathered, int rank,
                                                    const int32_t* __restrict__ plan, __nv_bfloat16* snap,
                                                    int nslots, float* Sfinal, int B, int d, int F) {
  __shared__ float4 s_in[32][33];
  __shared__ float4 s_fin[32][33];
  const int ntn = F / 128;
  const int q = blockIdx.x & 3;
  const int tile_all = blockIdx.x >> 2;
  const int per_row = (d / 128) * ntn;
  const int b = tile_all / per_row;
  const int tile = tile_all % per_row;
  const int mt = tile / ntn, nt = tile % ntn;
  const int j0 = plan[B + b], pre = plan[2 * B + b], keep = plan[3 * B + b];
  const size_t per = (size_t)d * F;
  const size_t tbase = (size_t)b * per + (size_t)tile * 16384;
  const int r = threadIdx.x & 31;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int g = (threadIdx.x >> 5) + 8 * it;  // 4-column group of the tile
    const size_t idx = tbase + ((size_t)g * 128 + q * 32 + r) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = j0; j < rank; ++j) {
      const float4 v = *reinterpret_cast<const float4*>(gathered + (size_t)j * B * per + idx);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    s_in[r][g] = acc;
    if (Sfinal) {
      float4 a = *reinterpret_cast<const float4*>(gathered + (size_t)rank * B * per + idx);
      if (keep) {
        a.x += acc.x;
        a.y += acc.y;
        a.z += acc.z;
        a.w += acc.w;
      }
      s_fin[r][g] = a;
    }
  }
  __syncthreads();
  const int wr = threadIdx.x >> 3;   // tile row of the quarter
  const int part = threadIdx.x & 7;  // 16 columns
  const size_t grow = (size_t)mt * 128 + q * 32 + wr;
  const size_t gcol = (size_t)nt * 128 + part * 16;
  if (Sfinal) {
    float4* dst = reinterpret_cast<float4*>(Sfinal + (size_t)b * per + grow * F + gcol);
#pragma unroll
    for (int u = 0; u < 4; ++u) dst[u] = s_fin[wr][part * 4 + u];
  }
  if (pre <= 0) return;
  float add[16];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float4 v = s_in[wr][part * 4 + u];
    add[4 * u] = v.x;
    add[4 * u + 1] = v.y;
    add[4 * u + 2] = v.z;
    add[4 * u + 3] = v.w;
  }
  for (int i = 0; i < pre; ++i) {
    uint4* p = reinterpret_cast<uint4*>(snap + ((size_t)(i % nslots) * B + b) * per + grow * F + gcol);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 w = p[h];
      uint32_t* e = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        __nv_bfloat162 v2 = *reinterpret_cast<__nv_bfloat162*>(&e[x]);
        const float lo = __low2float(v2) + add[8 * h + 2 * x];
        const float hi = __high2float(v2) + add[8 * h + 2 * x + 1];
        v2 = __floats2bfloat162_rn(lo, hi);
        e[x] = *reinterpret_cast<uint32_t*>(&v2);
      }
      p[h] = w;
    }
  }
}

cudaError_t cp_combine(const float* gathered, int world, int rank, const int32_t* plan, void* snap, int nslots,
                       float* Sfinal, const Shape& s, cudaStream_t st) {
  if (rank < 0 || rank >= world || s.d % 128 != 0 || s.F % 128 != 0) return cudaErrorInvalidValue;
  const long long blocks = (long long)s.B * (s.d / 128) * (s.F / 128) * 4;
  if (blocks <= 0 || blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  k_cp_combine<<<(unsigned)blocks, 256, 0, st>>>(gathered, rank, plan, (__nv_bfloat16*)snap, nslots, Sfinal, s.B,
                                                 s.d, s.F);
  return cudaGetLastError();
}

// Streaming bookkeeping: every row has now consumed `T` more tokens.
__global__ void k_stream_advance(long long* pos, int32_t* cont, int B, int T) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) {
    pos[b] += T;
    cont[b] = 1;
  }
}

cudaError_t stream_advance(long long* pos, int32_t* cont, int B, int T, cudaStream_t st) {
  k_stream_advance<<<(B + 127) / 128, 128, 0, st>>>(pos, cont, B, T);
  return cudaGetLastError();
}

}  // namespace aux
}  // namespace ipttt

namespace ipttt {
namespace aux {

// V[b,t,:] *= alpha[b, chunk(t)] * eta, in place (bf16), so that the state update's
// MMAs accumulate alpha eta V^T Z directly.
__global__ void k_prescale(__nv_bfloat16* V, const float* alpha, int B, int Tn, int d, int C, int k, float eta) {
  const int groups = d / 8;
  const size_t total = (size_t)B * Tn * groups;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const size_t bt = i / groups;
    const int t = (int)(bt % Tn);
    const int b = (int)(bt / Tn);
    const float sc = alpha[(size_t)b * k + t / C] * eta;
    __nv_bfloat16* v = V + bt * d + (size_t)(i % groups) * 8;
    float x[8];
    load_vec<__nv_bfloat16, 8>(v, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] *= sc;
    store_vec<__nv_bfloat16, 8>(v, x);
  }
}

// One block per (row, group of blockDim.x tokens): thread i holds token g0 + i; an
// inclusive max-scan of (start flag ? i : 0) gives the offset of the last document
// start at or before the token inside the group (0 if none).
__global__ void __launch_bounds__(1024) k_group_lo(const uint8_t* flags, uint16_t* glo, int Tn, int groups) {
  __shared__ int wmax[32];
  const int b = blockIdx.x / groups, g = blockIdx.x % groups;
  const int i = threadIdx.x, t = g * blockDim.x + i;
  const int lane = i & 31, w = i >> 5;
  int v = (t < Tn && flags[(size_t)b * Tn + t]) ? i : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v = max(v, u);
  }
  if (lane == 31) wmax[w] = v;
  __syncthreads();
  int pre = 0;
  for (int q = 0; q < w; ++q) pre = max(pre, wmax[q]);
  v = max(v, pre);
  if (t < Tn) glo[(size_t)b * Tn + t] = (uint16_t)v;
}

cudaError_t group_meta(const uint8_t* flags, ChunkMeta* gmeta, uint16_t* glo, const Shape& gs, cudaStream_t st) {
  if (gs.C % 32 != 0 || gs.C > 1024) return cudaErrorInvalidValue;
  k_chunk_meta<<<gs.B * gs.k, 256, 0, st>>>(flags, gmeta, gs.B, gs.T, gs.C, gs.k);
  k_group_lo<<<gs.B * gs.k, gs.C, 0, st>>>(flags, glo, gs.T, gs.k);
  return cudaGetLastError();
}

cudaError_t prescale_target(void* V, const float* alpha, const Shape& s, float eta, cudaStream_t st) {
  k_prescale<<<148 * 8, 256, 0, st>>>((__nv_bfloat16*)V, alpha, s.B, s.T, s.d, s.C, s.k, eta);
  return cudaGetLastError();
}

}  // namespace aux
}  // namespace ipttt
