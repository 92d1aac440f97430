// Backward of the In-Place TTT MLP layer: the fp32 gradients of
//   L = <gO, O> + <gS, S_final>
// with respect to H, X0, Wgate, Wup, Wdown0, conv_w and Wtarget, for either dtype
// (bf16 inputs are widened to fp32 first; every product runs in fp32 on the
// CUDA cores, with the strided GEMM of the all-fp32 forward).
//
// The pages give the forward only, and the layer is trained in place (continual
// training of the inserted conv and projection: cloud.tencent.com "榨干MLP的剩余价值",
// 验证模块一); the gradients follow by the chain rule through the forward of
// lijianxiong.blog notes "In-Place Test-Time Training", 方法 (gated MLP, apply,
// Hebbian update, LM-aligned target), the clip of 详细步骤 4 and the exclusive scan
// with document resets of the iplexlaw.co.kr review, §3 and §6.  Per row, with
// A = H Wg^T, Bu = H Wu^T, Z = SiLU(A) * Bu, U = masked conv(X0), V = U Wt, and per
// chunk i (first segment F_i continuing the previous chunk's document when cont_i,
// last segment L_i), P_i = V_L^T Z_L, dW_i = a_i eta P_i:
//   gW0 = gO^T Z;   gZ = gO W0;   g = gS (dL/dS after the last chunk)
//   for i = k-1 .. 0:
//     gP = eta g                                     (the delta was not clipped)
//        = tau/|P| g - tau <P, g>/|P|^3 P            (clipped to norm tau)
//     gV_L += Z_L gP^T;   gZ_L += V_L gP
//     gZ_F += gO_F S_i;   g = (keep_i ? g : 0) + gO_F^T Z_F
//   gA = gZ Bu SiLU'(A);  gBu = gZ SiLU(A)
//   gH = gA Wg + gBu Wu;  gWg = gA^T H;  gWu = gBu^T H
//   gU = gV Wt^T;  gWt = U^T gV;  conv: gX0[t+o] += w[o] gU[t] m(t,o), gw[o] += X0[t+o] gU[t] m(t,o)
// S_i (the state chunk i is applied with) is kept for every chunk from a forward
// pass over the chunks.  Deterministic: no atomics; reductions in a fixed order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <algorithm>

#include "aux_kernels.h"
#include "common.cuh"
#include "gemm.h"
#include "tc_kernels.h"

namespace ipttt {
namespace bwd {

namespace {

constexpr int kTaps = 5;
constexpr int kRedBlocks = 64;  // per-row partial sums of the norm and dot reductions

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

__global__ void k_widen(const __nv_bfloat16* __restrict__ in, float* __restrict__ out, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    out[i] = __bfloat162float(in[i]);
}

// Z = SiLU(A) * Bu
__global__ void k_gate(const float* A, const float* Bu, float* Z, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    Z[i] = silu_precise(A[i]) * Bu[i];
}

// gA = gZ Bu SiLU'(A), gBu = gZ SiLU(A), in place of A and Bu;
// SiLU'(x) = s(x) (1 + x (1 - s(x))), s the logistic function.
__global__ void k_gate_backward(float* A, float* Bu, const float* gZ, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float a = A[i], u = Bu[i], g = gZ[i];
    const float s = 1.0f / (1.0f + expf(-a));
    A[i] = g * u * (s * (1.0f + a * (1.0f - s)));
    Bu[i] = g * (a * s);
  }
}

// gO restricted to the first segment of each chunk that continues a document
// (the rows that read the carried state); zero elsewhere.
__global__ void k_first_segment(const float* gO, float* gOF, const ChunkMeta* meta, int B, int T, int d, int C,
                                int k) {
  const size_t n = (size_t)B * T * d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t bt = i / d;
    const int t = (int)(bt % T), b = (int)(bt / T);
    const ChunkMeta m = meta[(size_t)b * k + t / C];
    gOF[i] = (m.cont && t < m.first_end) ? gO[i] : 0.0f;
  }
}

// Per row b: partial sums over blocks of x.y (and of x.x) of the [n] slices, fp64.
__global__ void k_dot_partials(const float* x, const float* y, size_t n, double* part_xy, double* part_xx) {
  __shared__ double s1[256], s2[256];
  const int b = blockIdx.y;
  const float* xb = x + b * n;
  const float* yb = y + b * n;
  double a = 0.0, c = 0.0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    a += (double)xb[i] * (double)yb[i];
    c += (double)xb[i] * (double)xb[i];
  }
  s1[threadIdx.x] = a;
  s2[threadIdx.x] = c;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      s1[threadIdx.x] += s1[threadIdx.x + o];
      s2[threadIdx.x] += s2[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    part_xy[(size_t)b * gridDim.x + blockIdx.x] = s1[0];
    part_xx[(size_t)b * gridDim.x + blockIdx.x] = s2[0];
  }
}

// Per row b, from |P|^2 and <P, g>: the coefficients of gP = c1 g + c2 P.
__global__ void k_clip_coeffs(const double* part_pg, const double* part_pp, int nblk, float* c12, int B, float eta,
                              float tau) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  double pg = 0.0, pp = 0.0;
  for (int q = 0; q < nblk; ++q) {
    pg += part_pg[(size_t)b * nblk + q];
    pp += part_pp[(size_t)b * nblk + q];
  }
  const double pn = sqrt(fmax(pp, 0.0));
  const bool clipped = tau > 0.0f && isfinite(tau) && (double)eta * pn > (double)tau;
  c12[2 * b] = clipped ? (float)(tau / pn) : eta;
  c12[2 * b + 1] = clipped ? (float)(-(double)tau * pg / (pn * pn * pn)) : 0.0f;
}

// gP = c1 g + c2 P per row b.
__global__ void k_grad_delta(const float* g, const float* P, float* gP, const float* c12, size_t n) {
  const int b = blockIdx.y;
  const float c1 = c12[2 * b], c2 = c12[2 * b + 1];
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    gP[b * n + i] = fmaf(c1, g[b * n + i], c2 * P[b * n + i]);
}

// g = (chunk holds a document start ? 0 : g) + raw, per row b.
__global__ void k_carry_back(float* g, const float* raw, size_t n, const ChunkMeta* meta, int k, int chunk) {
  const int b = blockIdx.y;
  const bool keep = !meta[(size_t)b * k + chunk].has_start;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    g[b * n + i] = (keep ? g[b * n + i] : 0.0f) + raw[b * n + i];
}

// Number of taps in use at token t (tap o and later are dropped once t+o reaches
// the chunk end, T, or a document start).
__device__ __forceinline__ int taps_at(const uint8_t* f, int t, int T, int C) {
  const int cend = min((t / C + 1) * C, T);
  int n = 1;
  for (int o = 1; o < kTaps; ++o)
    if (n == o && t + o < cend && !f[t + o]) n = o + 1;
  return n;
}

// gX0[s, c] = sum_o w[c, o] gU[s - o, c] over the taps o in use at token s - o.
__global__ void k_conv_grad_input(const float* gU, const float* cw, const uint8_t* flags, float* gX0, int B, int T,
                                  int d, int C) {
  const size_t n = (size_t)B * T * d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % d);
    const size_t bt = i / d;
    const int s = (int)(bt % T), b = (int)(bt / T);
    const uint8_t* f = flags + (size_t)b * T;
    float acc = 0.0f;
    for (int o = 0; o < kTaps; ++o) {
      const int t = s - o;
      if (t < 0) break;
      if (o < taps_at(f, t, T, C)) acc = fmaf(cw[c * kTaps + o], gU[((size_t)b * T + t) * d + c], acc);
    }
    gX0[i] = acc;
  }
}

// gw[c, o] = sum over rows b and tokens t of X0[t + o, c] gU[t, c] over the taps in
// use: one block per (c, o), a fixed-order reduction.
__global__ void k_conv_grad_weight(const float* gU, const float* X0, const uint8_t* flags, float* gw, int B, int T,
                                   int d, int C) {
  __shared__ double sh[256];
  const int c = blockIdx.x / kTaps, o = blockIdx.x % kTaps;
  double acc = 0.0;
  for (size_t bt = threadIdx.x; bt < (size_t)B * T; bt += blockDim.x) {
    const int t = (int)(bt % T), b = (int)(bt / T);
    if (o < taps_at(flags + (size_t)b * T, t, T, C))
      acc += (double)X0[((size_t)b * T + t + o) * d + c] * (double)gU[bt * d + c];
  }
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) gw[c * kTaps + o] = (float)sh[0];
}

unsigned grid_for(size_t n) { return (unsigned)std::min<size_t>((n + 255) / 256, 148 * 16); }
// Kernels with one token per block iteration and threads over w channel groups:
// blocks of w threads rounded up to a warp (at most 1024), as many as fit on the
// SMs at once (at most one per token).
unsigned token_block(long long w) { return (unsigned)std::min<long long>(1024, (w + 31) / 32 * 32); }
unsigned token_grid(long long tokens, long long w) {
  const long long per_sm = std::max<long long>(1, 2048 / token_block(w));
  return (unsigned)std::max<long long>(1, std::min<long long>(tokens, 148 * per_sm));
}

}  // namespace

struct BwdLayout {
  size_t flags, meta, alpha, dpart, part1, part2, c12, H, X0, gO, Wg, Wu, W0, cw, Wt, A, Bu, Z, U, V, gZ, gV, gOF,
      states, P, g, gP, raw, total;
};

BwdLayout bwd_layout(const Shape& s) {
  const size_t B = s.B, T = s.T, d = s.d, F = s.F, k = s.k;
  BwdLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += al256(bytes);
    return o;
  };
  L.flags = take(B * T);
  L.meta = take(B * k * sizeof(ChunkMeta));
  L.alpha = take(B * k * 4);
  L.dpart = take(B * 64 * sizeof(double));
  L.part1 = take(B * kRedBlocks * sizeof(double));
  L.part2 = take(B * kRedBlocks * sizeof(double));
  L.c12 = take(B * 2 * 4);
  L.H = take(B * T * d * 4);
  L.X0 = take(B * T * d * 4);
  L.gO = take(B * T * d * 4);
  L.Wg = take(F * d * 4);
  L.Wu = take(F * d * 4);
  L.W0 = take(d * F * 4);
  L.cw = take(d * kTaps * 4);
  L.Wt = take(d * d * 4);
  L.A = take(B * T * F * 4);
  L.Bu = take(B * T * F * 4);
  L.Z = take(B * T * F * 4);
  L.U = take(B * T * d * 4);
  L.V = take(B * T * d * 4);
  L.gZ = take(B * T * F * 4);
  L.gV = take(B * T * d * 4);
  L.gOF = take(B * T * d * 4);
  L.states = take(k * B * d * F * 4);
  L.P = take(B * d * F * 4);
  L.g = take(B * d * F * 4);
  L.gP = take(B * d * F * 4);
  L.raw = take(B * d * F * 4);
  L.total = off;
  return L;
}

size_t workspace_bytes(const Shape& s) { return bwd_layout(s).total; }

// Kernels one call launches: the widening of its 8 inputs (bf16 only), 20 outside
// the chunk loops (3 of them the document metadata), and per chunk 4 in the
// forward recompute and 9 in the reverse scan.
long long launches(const Shape& s, int dtype) { return (dtype == IPTTT_BF16 ? 8 : 0) + 20 + 13LL * s.k; }

#define BW_CHECK(expr)                                 \
  do {                                                 \
    cudaError_t e_ = (expr);                           \
    if (e_ != cudaSuccess) return e_;                  \
  } while (0)

cudaError_t run(const Shape& s, int dtype, float eta, float tau, const void* H_, const void* X0_, const void* Wg_,
                const void* Wu_, const void* W0_, const void* cw_, const void* Wt_, const int32_t* doc, int n_doc,
                const void* gO_, const float* gS, float* gH, float* gX0, float* gWg, float* gWu, float* gW0,
                float* gcw, float* gWt, uint8_t* ws, int* status, cudaStream_t st) {
  using namespace aux;
  const BwdLayout L = bwd_layout(s);
  const long long B = s.B, T = s.T, d = s.d, F = s.F;
  const int k = s.k;
  uint8_t* flags = ws + L.flags;
  ChunkMeta* meta = reinterpret_cast<ChunkMeta*>(ws + L.meta);
  float* alpha = reinterpret_cast<float*>(ws + L.alpha);
  double* dpart = reinterpret_cast<double*>(ws + L.dpart);
  double* p1 = reinterpret_cast<double*>(ws + L.part1);
  double* p2 = reinterpret_cast<double*>(ws + L.part2);
  float* c12 = reinterpret_cast<float*>(ws + L.c12);
  auto fp = [&](size_t o) { return reinterpret_cast<float*>(ws + o); };
  float *H = fp(L.H), *X0 = fp(L.X0), *gO = fp(L.gO), *Wg = fp(L.Wg), *Wu = fp(L.Wu), *W0 = fp(L.W0),
        *cw = fp(L.cw), *Wt = fp(L.Wt), *A = fp(L.A), *Bu = fp(L.Bu), *Z = fp(L.Z), *U = fp(L.U), *V = fp(L.V),
        *gZ = fp(L.gZ), *gV = fp(L.gV), *gOF = fp(L.gOF), *states = fp(L.states), *P = fp(L.P), *g = fp(L.g),
        *gP = fp(L.gP), *raw = fp(L.raw);
  const size_t nS = (size_t)d * F;

  // inputs in fp32
  struct In { const void* src; float* dst; size_t n; };
  const In ins[] = {{H_, H, (size_t)(B * T * d)}, {X0_, X0, (size_t)(B * T * d)}, {gO_, gO, (size_t)(B * T * d)},
                    {Wg_, Wg, (size_t)(F * d)}, {Wu_, Wu, (size_t)(F * d)}, {W0_, W0, (size_t)(d * F)},
                    {cw_, cw, (size_t)(d * kTaps)}, {Wt_, Wt, (size_t)(d * d)}};
  for (const In& in : ins) {
    if (dtype == IPTTT_BF16)
      k_widen<<<grid_for(in.n), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(in.src), in.dst, in.n);
    else
      BW_CHECK(cudaMemcpyAsync(in.dst, in.src, in.n * 4, cudaMemcpyDeviceToDevice, st));
  }
  BW_CHECK(build_meta(flags, meta, s, doc, n_doc, nullptr, status, st));

  // forward recompute: A, Bu, Z, U, V (last-segment rows), states S_i
  SimtArgs a{};
  a.M = (int)T; a.N = (int)F; a.K = (int)d;
  a.A = H; a.sam = d; a.sak = 1; a.sab = T * d;
  a.B0 = Wg; a.s0n = d; a.s0k = 1; a.s0b = 0;
  a.mode = SM_RAW;
  a.out = A; a.som = F; a.son = 1; a.sob = T * F;
  BW_CHECK(simt_gemm(a, (int)B, st));
  a.B0 = Wu; a.out = Bu;
  BW_CHECK(simt_gemm(a, (int)B, st));
  k_gate<<<grid_for(B * T * F), 256, 0, st>>>(A, Bu, Z, (size_t)(B * T * F));
  BW_CHECK(conv_target(IPTTT_F32, X0, cw, flags, U, s, st));
  SimtArgs v{};
  v.M = (int)T; v.N = (int)d; v.K = (int)d;
  v.A = U; v.sam = d; v.sak = 1; v.sab = T * d;
  v.B0 = Wt; v.s0n = 1; v.s0k = d; v.s0b = 0;
  v.mode = SM_V;
  v.out = V; v.som = d; v.son = 1; v.sob = T * d;
  v.meta = meta; v.k = k; v.C = s.C; v.row0 = 0;
  BW_CHECK(simt_gemm(v, (int)B, st));
  BW_CHECK(cudaMemsetAsync(g, 0, B * nS * 4, st));  // the forward state, then the backward carry
  for (int i = 0; i < k; ++i) {
    const long long t0 = (long long)i * s.C;
    const int rows = (int)std::min<long long>(s.C, T - t0);
    BW_CHECK(cudaMemcpyAsync(states + (size_t)i * B * nS, g, B * nS * 4, cudaMemcpyDeviceToDevice, st));
    SimtArgs r{};
    r.M = (int)d; r.N = (int)F; r.K = rows;
    r.A = V + t0 * d; r.sam = 1; r.sak = d; r.sab = T * d;
    r.B0 = Z + t0 * F; r.s0n = 1; r.s0k = F; r.s0b = T * F;
    r.mode = SM_RAW;
    r.out = raw; r.som = F; r.son = 1; r.sob = nS;
    BW_CHECK(simt_gemm(r, (int)B, st));
    BW_CHECK(simt_update_state(g, raw, dpart, alpha, meta, s, i, eta, tau, st));
  }

  // gW0 = gO^T Z over every row and token
  SimtArgs w0{};
  w0.M = (int)d; w0.N = (int)F; w0.K = (int)(B * T);
  w0.A = gO; w0.sam = 1; w0.sak = d; w0.sab = 0;
  w0.B0 = Z; w0.s0n = 1; w0.s0k = F; w0.s0b = 0;
  w0.mode = SM_RAW;
  w0.out = gW0; w0.som = F; w0.son = 1; w0.sob = 0;
  BW_CHECK(simt_gemm(w0, 1, st));
  // gZ = gO W0
  SimtArgs gz{};
  gz.M = (int)T; gz.N = (int)F; gz.K = (int)d;
  gz.A = gO; gz.sam = d; gz.sak = 1; gz.sab = T * d;
  gz.B0 = W0; gz.s0n = 1; gz.s0k = F; gz.s0b = 0;
  gz.mode = SM_RAW;
  gz.out = gZ; gz.som = F; gz.son = 1; gz.sob = T * F;
  BW_CHECK(simt_gemm(gz, (int)B, st));
  k_first_segment<<<grid_for(B * T * d), 256, 0, st>>>(gO, gOF, meta, (int)B, (int)T, (int)d, s.C, k);
  BW_CHECK(cudaMemsetAsync(gV, 0, B * T * d * 4, st));

  // reverse scan over the chunks
  if (gS)
    BW_CHECK(cudaMemcpyAsync(g, gS, B * nS * 4, cudaMemcpyDeviceToDevice, st));
  else
    BW_CHECK(cudaMemsetAsync(g, 0, B * nS * 4, st));
  const dim3 rgrid(kRedBlocks, (unsigned)B);
  const dim3 egrid((unsigned)std::min<size_t>((nS + 255) / 256, 1024), (unsigned)B);
  for (int i = k - 1; i >= 0; --i) {
    const long long t0 = (long long)i * s.C;
    const int rows = (int)std::min<long long>(s.C, T - t0);
    // P_i = V_L^T Z_L (V is zero outside the last segment)
    SimtArgs r{};
    r.M = (int)d; r.N = (int)F; r.K = rows;
    r.A = V + t0 * d; r.sam = 1; r.sak = d; r.sab = T * d;
    r.B0 = Z + t0 * F; r.s0n = 1; r.s0k = F; r.s0b = T * F;
    r.mode = SM_RAW;
    r.out = P; r.som = F; r.son = 1; r.sob = nS;
    BW_CHECK(simt_gemm(r, (int)B, st));
    k_dot_partials<<<rgrid, 256, 0, st>>>(P, g, nS, p1, p2);
    k_clip_coeffs<<<((unsigned)B + 127) / 128, 128, 0, st>>>(p1, p2, kRedBlocks, c12, (int)B, eta, tau);
    k_grad_delta<<<egrid, 256, 0, st>>>(g, P, gP, c12, nS);
    // gV_L += Z_L gP^T (rows of the last segment)
    SimtArgs gv{};
    gv.M = rows; gv.N = (int)d; gv.K = (int)F;
    gv.A = Z + t0 * F; gv.sam = F; gv.sak = 1; gv.sab = T * F;
    gv.B0 = gP; gv.s0n = F; gv.s0k = 1; gv.s0b = nS;
    gv.mode = SM_ACC_L;
    gv.out = gV + t0 * d; gv.som = d; gv.son = 1; gv.sob = T * d;
    gv.meta = meta; gv.k = k; gv.C = s.C; gv.row0 = (int)t0;
    BW_CHECK(simt_gemm(gv, (int)B, st));
    // gZ_L += V_L gP (V is zero outside the last segment)
    SimtArgs gzl{};
    gzl.M = rows; gzl.N = (int)F; gzl.K = (int)d;
    gzl.A = V + t0 * d; gzl.sam = d; gzl.sak = 1; gzl.sab = T * d;
    gzl.B0 = gP; gzl.s0n = 1; gzl.s0k = F; gzl.s0b = nS;
    gzl.mode = SM_ACC;
    gzl.out = gZ + t0 * F; gzl.som = F; gzl.son = 1; gzl.sob = T * F;
    BW_CHECK(simt_gemm(gzl, (int)B, st));
    // gZ_F += gO_F S_i (gO_F is zero outside the continuing first segment)
    SimtArgs gzf = gzl;
    gzf.A = gOF + t0 * d;
    gzf.B0 = states + (size_t)i * B * nS; gzf.s0b = nS;
    BW_CHECK(simt_gemm(gzf, (int)B, st));
    // g = (keep ? g : 0) + gO_F^T Z_F
    SimtArgs gr{};
    gr.M = (int)d; gr.N = (int)F; gr.K = rows;
    gr.A = gOF + t0 * d; gr.sam = 1; gr.sak = d; gr.sab = T * d;
    gr.B0 = Z + t0 * F; gr.s0n = 1; gr.s0k = F; gr.s0b = T * F;
    gr.mode = SM_RAW;
    gr.out = raw; gr.som = F; gr.son = 1; gr.sob = nS;
    BW_CHECK(simt_gemm(gr, (int)B, st));
    k_carry_back<<<egrid, 256, 0, st>>>(g, raw, nS, meta, k, i);
  }

  // the gated activation, then H and the gate/up weights
  k_gate_backward<<<grid_for(B * T * F), 256, 0, st>>>(A, Bu, gZ, (size_t)(B * T * F));
  SimtArgs gh{};
  gh.M = (int)T; gh.N = (int)d; gh.K = (int)F;
  gh.A = A; gh.sam = F; gh.sak = 1; gh.sab = T * F;
  gh.B0 = Wg; gh.s0n = 1; gh.s0k = d; gh.s0b = 0;
  gh.mode = SM_RAW;
  gh.out = gH; gh.som = d; gh.son = 1; gh.sob = T * d;
  BW_CHECK(simt_gemm(gh, (int)B, st));
  gh.A = Bu; gh.B0 = Wu; gh.mode = SM_ACC;
  BW_CHECK(simt_gemm(gh, (int)B, st));
  SimtArgs gw{};
  gw.M = (int)F; gw.N = (int)d; gw.K = (int)(B * T);
  gw.A = A; gw.sam = 1; gw.sak = F; gw.sab = 0;
  gw.B0 = H; gw.s0n = 1; gw.s0k = d; gw.s0b = 0;
  gw.mode = SM_RAW;
  gw.out = gWg; gw.som = d; gw.son = 1; gw.sob = 0;
  BW_CHECK(simt_gemm(gw, 1, st));
  gw.A = Bu; gw.out = gWu;
  BW_CHECK(simt_gemm(gw, 1, st));

  // the target: gU = gV Wt^T (into V's buffer, no longer needed), gWt = U^T gV, then the conv
  float* gU = V;
  SimtArgs gu{};
  gu.M = (int)T; gu.N = (int)d; gu.K = (int)d;
  gu.A = gV; gu.sam = d; gu.sak = 1; gu.sab = T * d;
  gu.B0 = Wt; gu.s0n = d; gu.s0k = 1; gu.s0b = 0;
  gu.mode = SM_RAW;
  gu.out = gU; gu.som = d; gu.son = 1; gu.sob = T * d;
  BW_CHECK(simt_gemm(gu, (int)B, st));
  SimtArgs gt{};
  gt.M = (int)d; gt.N = (int)d; gt.K = (int)(B * T);
  gt.A = U; gt.sam = 1; gt.sak = d; gt.sab = 0;
  gt.B0 = gV; gt.s0n = 1; gt.s0k = d; gt.s0b = 0;
  gt.mode = SM_RAW;
  gt.out = gWt; gt.som = d; gt.son = 1; gt.sob = 0;
  BW_CHECK(simt_gemm(gt, 1, st));
  k_conv_grad_input<<<grid_for(B * T * d), 256, 0, st>>>(gU, cw, flags, gX0, (int)B, (int)T, (int)d, s.C);
  k_conv_grad_weight<<<(unsigned)(d * kTaps), 256, 0, st>>>(gU, X0, flags, gcw, (int)B, (int)T, (int)d, s.C);
  return cudaGetLastError();
}


// ------------------------------------------------------------------ bf16 path, tensor cores
// The same gradients on the bf16 path, every product a tcgen05 GEMM (gemm.cu)
// on bf16 operands with fp32 accumulators, from the forward's own Z, U, V, clip
// factors and per-chunk state copies S_i (run beforehand into the workspace with
// every S_i kept).  With P_i = V_L^T Z_L (the raw delta of chunk i), G_i = dL/dS_i:
//   G_k = gS;  G_i = keep_i G_{i+1} + gO_F^T Z_F            (reverse scan, fp32; bf16 copies of G_{i+1})
//   the delta alpha_i eta P_i gets gP = c1 G_{i+1} + c2 P_i with c1 = alpha_i eta and, for a
//   clipped chunk (alpha_i < 1, so ||P_i|| = tau / (alpha_i eta)),
//   c2 = -tau <P_i, G_{i+1}> / ||P_i||^3 = -alpha_i^3 eta^3 <P_i, G_{i+1}> / tau^2, else 0;
//   <P_i, G_{i+1}> = sum_{t in L} v_t . (G_{i+1} z_t) = sum_t v_t . Y_t,  Y = Z G_{i+1}^T
//   gV_L = c1 Y + c2 Z_L P_i^T;  gZ = gO W0 + c1 V_L G_{i+1} + c2 V_L P_i + gO_F S_i
//   then the gated activation, gH, gWgate, gWup, the target GEMM and the conv as on the fp32 path.
namespace {

// gO on the continued first segment of each chunk, zero elsewhere; 8 channels of
// one token per thread (d % 8 == 0, 16-byte rows).
__global__ void k_mask_first_bf16(const __nv_bfloat16* gO, __nv_bfloat16* gOF, const ChunkMeta* meta, int B, int T,
                                  int d, int C, int k) {
  const int g8 = d / 8;
  const size_t n = (size_t)B * T * g8;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t bt = i / g8;
    const int t = (int)(bt % T), b = (int)(bt / T);
    const ChunkMeta m = meta[(size_t)b * k + t / C];
    const bool keep = m.cont && t < m.first_end;
    reinterpret_cast<uint4*>(gOF)[i] = keep ? reinterpret_cast<const uint4*>(gO)[i] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// <P_i, G_{i+1}> = sum over the tokens of chunk i of v_t . Y_t (V is zero outside
// the last segment), as kDotParts fixed-order partial sums per (row, chunk) ...
constexpr int kDotParts = 32;
__global__ void k_vy_partials(const __nv_bfloat16* V, const float* Y, double* part, int T, int d, int C, int k) {
  __shared__ double sh[256];
  const int i = blockIdx.x, b = blockIdx.y, q = blockIdx.z;
  const int t0 = i * C, t1 = min(t0 + C, T);
  const size_t n = (size_t)(t1 - t0) * d;
  const size_t lo = n * q / kDotParts, hi = n * (q + 1) / kDotParts;
  const __nv_bfloat16* v = V + ((size_t)b * T + t0) * d;
  const float* y = Y + ((size_t)b * T + t0) * d;
  double acc = 0.0;
  for (size_t e = lo + threadIdx.x; e < hi; e += blockDim.x) acc += (double)__bfloat162float(v[e]) * (double)y[e];
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[((size_t)b * k + i) * kDotParts + q] = sh[0];
}

// ... then per (row b, chunk i): c1 = alpha eta, and c2 for a clipped chunk.
__global__ void k_clip_coeffs_tc(const double* part, const float* alpha, float* c1, float* c2, int n, float eta,
                                 float tau) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;  // b k + i
  if (j >= n) return;
  double dot = 0.0;
  for (int q = 0; q < kDotParts; ++q) dot += part[(size_t)j * kDotParts + q];
  const float a = alpha[j];
  c1[j] = a * eta;
  const bool clipped = tau > 0.0f && a < 1.0f;
  const double ae = (double)a * eta;
  c2[j] = clipped ? (float)(-ae * ae * ae * dot / ((double)tau * tau)) : 0.0f;
}

// gV = c1 Y on the rows of each chunk's last segment, 0 elsewhere.
__global__ void k_gv_init(const float* Y, const float* c1, float* gV, const ChunkMeta* meta, int B, int T, int d,
                          int C, int k) {
  // one token per block iteration (its chunk's row start and c1 read once), 4 channels per thread
  const int g4 = d / 4;
  const long long BT = (long long)B * T;
  for (long long bt = blockIdx.x; bt < BT; bt += gridDim.x) {
    const int t = (int)(bt % T);
    const size_t bi = (size_t)(bt / T) * k + t / C;
    const bool in_last = t >= meta[bi].last_start;
    const float sc = in_last ? c1[bi] : 0.0f;
    const float4* y = reinterpret_cast<const float4*>(Y + bt * d);
    float4* o = reinterpret_cast<float4*>(gV + bt * d);
    for (int c = threadIdx.x; c < g4; c += blockDim.x) {
      if (in_last) {
        const float4 v = y[c];
        o[c] = make_float4(sc * v.x, sc * v.y, sc * v.z, sc * v.w);
      } else {
        o[c] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
    }
  }
}

// gA = gZ Bu SiLU'(A), gBu = gZ SiLU(A), rounded to bf16 (the next products' operands);
// 8 elements per thread (n % 8 == 0).
__global__ void k_gate_backward_bf16(const __nv_bfloat16* A, const __nv_bfloat16* Bu, const float* gZ,
                                     __nv_bfloat16* gA, __nv_bfloat16* gBu, size_t n) {
  const size_t n8 = n / 8;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 av = reinterpret_cast<const uint4*>(A)[i], uv = reinterpret_cast<const uint4*>(Bu)[i];
    const float4 g0 = reinterpret_cast<const float4*>(gZ)[2 * i], g1 = reinterpret_cast<const float4*>(gZ)[2 * i + 1];
    const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    const __nv_bfloat162* ap = reinterpret_cast<const __nv_bfloat162*>(&av);
    const __nv_bfloat162* up = reinterpret_cast<const __nv_bfloat162*>(&uv);
    uint4 oa, ob;
    __nv_bfloat162* pa = reinterpret_cast<__nv_bfloat162*>(&oa);
    __nv_bfloat162* pb = reinterpret_cast<__nv_bfloat162*>(&ob);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a0 = __low2float(ap[q]), a1 = __high2float(ap[q]);
      const float u0 = __low2float(up[q]), u1 = __high2float(up[q]);
      const float s0 = 1.0f / (1.0f + expf(-a0)), s1 = 1.0f / (1.0f + expf(-a1));
      pa[q] = __floats2bfloat162_rn(g[2 * q] * u0 * (s0 * (1.0f + a0 * (1.0f - s0))),
                                    g[2 * q + 1] * u1 * (s1 * (1.0f + a1 * (1.0f - s1))));
      pb[q] = __floats2bfloat162_rn(g[2 * q] * (a0 * s0), g[2 * q + 1] * (a1 * s1));
    }
    reinterpret_cast<uint4*>(gA)[i] = oa;
    reinterpret_cast<uint4*>(gBu)[i] = ob;
  }
}

// gX0[s, c] = sum_o w[c, o] gU[s - o, c] over the taps o in use at token s - o.
// Threads over groups of 8 channels (d % 8 == 0), each holding its 8 x kTaps
// weights; blocks over tokens, the taps in use found once per token.
__global__ void k_conv_grad_input_v8(const float* gU, const float* cw, const uint8_t* flags, float* gX0, int B,
                                     int T, int d, int C) {
  const int g8 = d / 8;
  const long long BT = (long long)B * T;
  for (int c8 = threadIdx.x; c8 < g8; c8 += blockDim.x) {
    const int c0 = c8 * 8;
    float w[8 * kTaps];  // w[q * kTaps + o] = cw[c0 + q][o]: 40 consecutive floats, 16-byte aligned
    const float4* wv = reinterpret_cast<const float4*>(cw + (size_t)c0 * kTaps);
#pragma unroll
    for (int j = 0; j < 2 * kTaps; ++j) {
      const float4 x = wv[j];
      w[4 * j] = x.x; w[4 * j + 1] = x.y; w[4 * j + 2] = x.z; w[4 * j + 3] = x.w;
    }
    for (long long bt = blockIdx.x; bt < BT; bt += gridDim.x) {
      const int s = (int)(bt % T);
      const uint8_t* f = flags + (bt - s);
      float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int o = 0; o < kTaps; ++o) {
        const int t = s - o;
        if (t < 0 || o >= taps_at(f, t, T, C)) continue;
        const float4* u = reinterpret_cast<const float4*>(gU + (bt - o) * d + c0);
        const float4 u0 = u[0], u1 = u[1];
        const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(w[q * kTaps + o], uv[q], acc[q]);
      }
      float4* out = reinterpret_cast<float4*>(gX0 + bt * d + c0);
      out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// gw[c, o] = sum over rows and tokens of X0[t + o, c] gU[t, c] over the taps in
// use, in two fixed-order steps: block (channel block, part) sums a contiguous
// range of tokens for 256 channels (threads over channels, so loads are
// coalesced), then the parts are added in order.
constexpr int kConvParts = 256;
__global__ void k_conv_grad_weight_parts(const float* gU, const __nv_bfloat16* X0, const uint8_t* flags,
                                         float* part, int B, int T, int d, int C) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= d) return;
  const long long BT = (long long)B * T;
  const long long lo = BT * blockIdx.y / kConvParts, hi = BT * (blockIdx.y + 1) / kConvParts;
  float acc[kTaps] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  int t = (int)(lo % T);            // token and row of bt, advanced with it
  const uint8_t* f = flags + (lo - t);
#pragma unroll 4
  for (long long bt = lo; bt < hi; ++bt) {
    const float g = gU[bt * d + c];
    const int n = taps_at(f, t, T, C);
#pragma unroll
    for (int o = 0; o < kTaps; ++o)
      if (o < n) acc[o] = fmaf(__bfloat162float(X0[(bt + o) * d + c]), g, acc[o]);
    if (++t == T) {
      t = 0;
      f += T;
    }
  }
#pragma unroll
  for (int o = 0; o < kTaps; ++o) part[((size_t)blockIdx.y * d + c) * kTaps + o] = acc[o];
}

__global__ void k_conv_grad_weight_reduce(const float* part, float* gw, int d) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= d * kTaps) return;
  double s = 0.0;
  for (int q = 0; q < kConvParts; ++q) s += part[(size_t)q * d * kTaps + i];
  gw[i] = (float)s;
}

__global__ void k_f32_to_bf16(const float* x, __nv_bfloat16* y, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    y[i] = __float2bfloat16(x[i]);
}

struct TcLayout {
  size_t Af, Buf, gZ, gA, gBu, gOF, Y, gV, gVb, gU, P, G, Gs, c1, c2, dpart, cwf, cpart, total;
};

TcLayout tc_layout(const Shape& s) {
  const size_t B = s.B, T = s.T, d = s.d, F = s.F, k = s.k;
  TcLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += al256(bytes);
    return o;
  };
  L.Af = take(B * T * F * 2);
  L.Buf = take(B * T * F * 2);
  L.gZ = take(B * T * F * 4);
  L.gA = take(B * T * F * 2);
  L.gBu = take(B * T * F * 2);
  L.gOF = take(B * T * d * 2);
  L.Y = take(B * T * d * 4);
  L.gV = take(B * T * d * 4);
  L.gVb = take(B * T * d * 2);
  L.gU = take(B * T * d * 4);
  L.P = take(k * B * d * F * 2);
  L.G = take(B * d * F * 4);  // the reverse scan's fp32 state (blocked tiles)
  L.Gs = take(k * B * d * F * 2);
  L.c1 = take(B * k * 4);
  L.c2 = take(B * k * 4);
  L.dpart = take(B * k * kDotParts * sizeof(double));
  L.cwf = take(d * kTaps * 4);
  L.cpart = take((size_t)kConvParts * d * kTaps * 4);
  L.total = off;
  return L;
}


}  // namespace

size_t tc_workspace_bytes(const Shape& s) { return tc_layout(s).total; }

void* tc_delta_buffer(uint8_t* ws, const Shape& s) { return ws + tc_layout(s).P; }

// Kernels run_tc launches: 16 GEMMs (15 when the forward wrote the deltas), the
// reverse scan on the update kernel and 10 elementwise or reduction kernels, plus
// the state layout kernel when a gradient of the final state is given (a memset
// otherwise).
long long tc_launches(bool deltas_ready, bool has_gS) {
  return (deltas_ready ? 26 : 27) + (has_gS ? 1 : 0);
}


cudaError_t run_tc(const Shape& s, float eta, float tau, const TcForward& f, const void* H, const void* X0,
                   const void* Wg, const void* Wu, const void* W0, const void* cw, const void* Wt, const void* gO,
                   const float* gS, float* gH, float* gX0, float* gWg, float* gWu, float* gW0, float* gcw,
                   float* gWt, uint8_t* ws, int* status, int num_sms, cudaStream_t st) {
  using namespace gemm;
  const TcLayout L = tc_layout(s);
  const long long B = s.B, T = s.T, d = s.d, F = s.F;
  const int k = s.k;
  const uint64_t BT = (uint64_t)(B * T);
  auto fp = [&](size_t o) { return reinterpret_cast<float*>(ws + o); };
  auto hp = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(ws + o); };
  float *gZ = fp(L.gZ), *Y = fp(L.Y), *gV = fp(L.gV), *gU = fp(L.gU), *c1 = fp(L.c1), *c2 = fp(L.c2),
        *cwf = fp(L.cwf), *cpart = fp(L.cpart);
  double* dpart = reinterpret_cast<double*>(ws + L.dpart);
  __nv_bfloat16 *Af = hp(L.Af), *Buf = hp(L.Buf), *gA = hp(L.gA), *gBu = hp(L.gBu), *gOF = hp(L.gOF),
                *gVb = hp(L.gVb), *P = hp(L.P), *Gs = hp(L.Gs);
  const __nv_bfloat16* Zb = static_cast<const __nv_bfloat16*>(f.Z);
  const __nv_bfloat16* Vb = static_cast<const __nv_bfloat16*>(f.V);

  Args g{};
  g.status = status;
  auto plain = [&](int M, int N, int K, void* out, long long ldo, int kind) {
    g.mode = GM_PLAIN;
    g.M = M; g.N = N; g.K = K;
    g.out = out; g.ldo = ldo; g.osz = 0; g.out_kind = kind;
    g.scale = nullptr; g.meta = nullptr; g.rows = GR_ALL;
    return gemm::run(g, num_sms, st);
  };
  auto chunked = [&](int mode, int M, int N, int K, void* out, long long ldo, long long osz, int kind,
                     const float* scale, int rows, int nslots) {
    g.mode = mode;
    g.M = M; g.N = N; g.K = K;
    g.B = (int)B; g.T = (int)T; g.C = s.C; g.k = k;
    g.chunk0 = 0; g.nchunks = k; g.nslots = nslots;
    g.out = out; g.ldo = ldo; g.osz = osz; g.out_kind = kind;
    g.scale = scale; g.meta = f.meta; g.rows = rows;
    return gemm::run(g, num_sms, st);
  };

  // 1. pre-activations A = H Wg^T, Bu = H Wu^T (bf16)
  g.A = {H, (uint64_t)(d), (uint64_t)(BT), (uint64_t)(1)};
  g.Bop = {Wg, (uint64_t)(d), (uint64_t)(F), (uint64_t)(1)};
  g.a_mn = 0; g.b_mn = 0;
  BW_CHECK(plain((int)BT, (int)F, (int)d, Af, F, GO_BF16));
  g.Bop = {Wu, (uint64_t)(d), (uint64_t)(F), (uint64_t)(1)};
  BW_CHECK(plain((int)BT, (int)F, (int)d, Buf, F, GO_BF16));
  // 2. gZ = gO W0 (W0 [d][F]: k = d rows, n = F contiguous)
  g.A = {gO, (uint64_t)(d), (uint64_t)(BT), (uint64_t)(1)};
  g.Bop = {W0, (uint64_t)(F), (uint64_t)(d), (uint64_t)(1)};
  g.a_mn = 0; g.b_mn = 1;
  BW_CHECK(plain((int)BT, (int)F, (int)d, gZ, F, GO_F32));
  // 3. gW0 = gO^T Z over every token
  g.A = {gO, (uint64_t)(d), (uint64_t)(BT), (uint64_t)(1)};
  g.Bop = {Zb, (uint64_t)(F), (uint64_t)(BT), (uint64_t)(1)};
  g.a_mn = 1; g.b_mn = 1;
  BW_CHECK(plain((int)d, (int)F, (int)BT, gW0, F, GO_F32));
  // 4. P_i = V_L^T Z_L (unless the forward's state update wrote them); gO_F, gO on
  //    the continued first segment of each chunk
  g.A = {Vb, (uint64_t)(d), (uint64_t)(T), (uint64_t)(B)};
  g.Bop = {Zb, (uint64_t)(F), (uint64_t)(T), (uint64_t)(B)};
  if (!f.deltas_ready) BW_CHECK(chunked(GM_CHUNK_K, (int)d, (int)F, 0, P, F, d * F, GO_BF16, nullptr, GR_ALL, 1));
  k_mask_first_bf16<<<grid_for(B * T * d / 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(gO), gOF, f.meta, (int)B,
                                                          (int)T, (int)d, s.C, k);
  // 5. reverse scan on the state-update kernel: from G_k = gS, every chunk's
  //    gO_F^T Z_F formed from zero in TMEM and added in fp32 (registers), bf16 G_{i+1}
  //    into slot i of Gs before chunk i's term is added
  float* G = fp(L.G);
  BW_CHECK(aux::state_import_blocked(gS, G, s, st));
  {
    tck::TcParams q;
    memset(&q, 0, sizeof(q));
    q.B = (int)B; q.T = (int)T; q.d = (int)d; q.F = (int)F; q.C = s.C; q.k = k;
    q.meta = f.meta;
    q.S = G;
    q.status = status;
    q.nslots = k;
    q.chunk = 0;
    q.dchunks = k;
    q.upd_kb = tck::update_tokens_per_stage(s.C);
    q.n_tiles = (int)(B * (d / 128) * ((F + 255) / 256));
    q.rev = 1;
    if (!tck::make_map_bf16(&q.map[3], gOF, (uint64_t)d, (uint64_t)T, (uint64_t)B, 64, q.upd_kb) ||
        !tck::make_map_bf16(&q.map[4], Zb, (uint64_t)F, (uint64_t)T, (uint64_t)B, 64, q.upd_kb) ||
        !tck::make_map_bf16(&q.map[5], Gs, (uint64_t)F, (uint64_t)d, (uint64_t)k * B, 64, 32))
      return cudaErrorInvalidValue;
    BW_CHECK(tck::launch_update(q, num_sms, st));
  }
  // 6. Y = Z G_{i+1}^T on every chunk's tokens, then c1, c2 per chunk
  g.A = {Zb, (uint64_t)(F), (uint64_t)(T), (uint64_t)(B)};
  g.Bop = {Gs, (uint64_t)(F), (uint64_t)(d), (uint64_t)((uint64_t)k * B)};
  g.a_mn = 0; g.b_mn = 0;
  BW_CHECK(chunked(GM_CHUNK_ROWS, 0, (int)d, (int)F, Y, d, T * d, GO_F32, nullptr, GR_ALL, k));
  k_vy_partials<<<dim3(k, (unsigned)B, kDotParts), 256, 0, st>>>(Vb, Y, dpart, (int)T, (int)d, s.C, k);
  k_clip_coeffs_tc<<<(unsigned)((B * k + 127) / 128), 128, 0, st>>>(dpart, f.alpha, c1, c2, (int)(B * k), eta, tau);
  // 7. gV_L = c1 Y + c2 Z_L P_i^T
  k_gv_init<<<token_grid(BT, d / 4), token_block(d / 4), 0, st>>>(Y, c1, gV, f.meta, (int)B, (int)T, (int)d, s.C, k);
  g.Bop = {P, (uint64_t)(F), (uint64_t)(d), (uint64_t)((uint64_t)k * B)};
  BW_CHECK(chunked(GM_CHUNK_ROWS, 0, (int)d, (int)F, gV, d, T * d, GO_F32_ADD, c2, GR_LAST, k));
  // 8. gZ += c1 V_L G_{i+1} + c2 V_L P_i + gO_F S_i (K = d; the [d][F] operands n-major)
  g.A = {Vb, (uint64_t)(d), (uint64_t)(T), (uint64_t)(B)};
  g.Bop = {Gs, (uint64_t)(F), (uint64_t)(d), (uint64_t)((uint64_t)k * B)};
  g.a_mn = 0; g.b_mn = 1;
  BW_CHECK(chunked(GM_CHUNK_ROWS, 0, (int)F, (int)d, gZ, F, T * F, GO_F32_ADD, c1, GR_LAST, k));
  g.Bop = {P, (uint64_t)(F), (uint64_t)(d), (uint64_t)((uint64_t)k * B)};
  BW_CHECK(chunked(GM_CHUNK_ROWS, 0, (int)F, (int)d, gZ, F, T * F, GO_F32_ADD, c2, GR_LAST, k));
  g.A = {gO, (uint64_t)(d), (uint64_t)(T), (uint64_t)(B)};
  g.Bop = {f.snap, (uint64_t)(F), (uint64_t)(d), (uint64_t)((uint64_t)f.nslots * B)};
  BW_CHECK(chunked(GM_CHUNK_ROWS, 0, (int)F, (int)d, gZ, F, T * F, GO_F32_ADD, nullptr, GR_FIRST, f.nslots));
  // 9. the gated activation; gH = gA Wg + gBu Wu; gWg = gA^T H, gWu = gBu^T H
  k_gate_backward_bf16<<<grid_for(BT * F / 8), 256, 0, st>>>(Af, Buf, gZ, gA, gBu, (size_t)(BT * F));
  g.A = {gA, (uint64_t)(F), (uint64_t)(BT), (uint64_t)(1)};
  g.Bop = {Wg, (uint64_t)(d), (uint64_t)(F), (uint64_t)(1)};
  g.a_mn = 0; g.b_mn = 1;
  BW_CHECK(plain((int)BT, (int)d, (int)F, gH, d, GO_F32));
  g.A = {gBu, (uint64_t)(F), (uint64_t)(BT), (uint64_t)(1)};
  g.Bop = {Wu, (uint64_t)(d), (uint64_t)(F), (uint64_t)(1)};
  BW_CHECK(plain((int)BT, (int)d, (int)F, gH, d, GO_F32_ADD));
  g.A = {gA, (uint64_t)(F), (uint64_t)(BT), (uint64_t)(1)};
  g.Bop = {H, (uint64_t)(d), (uint64_t)(BT), (uint64_t)(1)};
  g.a_mn = 1; g.b_mn = 1;
  BW_CHECK(plain((int)F, (int)d, (int)BT, gWg, d, GO_F32));
  g.A = {gBu, (uint64_t)(F), (uint64_t)(BT), (uint64_t)(1)};
  BW_CHECK(plain((int)F, (int)d, (int)BT, gWu, d, GO_F32));
  // 10. the target: gU = gV Wt^T, gWt = U^T gV, then the conv
  k_f32_to_bf16<<<grid_for(BT * d), 256, 0, st>>>(gV, gVb, (size_t)(BT * d));
  g.A = {gVb, (uint64_t)(d), (uint64_t)(BT), (uint64_t)(1)};
  g.Bop = {Wt, (uint64_t)(d), (uint64_t)(d), (uint64_t)(1)};
  g.a_mn = 0; g.b_mn = 0;
  BW_CHECK(plain((int)BT, (int)d, (int)d, gU, d, GO_F32));
  g.A = {f.U, (uint64_t)(d), (uint64_t)(BT), (uint64_t)(1)};
  g.Bop = {gVb, (uint64_t)(d), (uint64_t)(BT), (uint64_t)(1)};
  g.a_mn = 1; g.b_mn = 1;
  BW_CHECK(plain((int)d, (int)d, (int)BT, gWt, d, GO_F32));
  k_widen<<<grid_for(d * kTaps), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(cw), cwf, (size_t)(d * kTaps));
  k_conv_grad_input_v8<<<token_grid(BT, d / 8), token_block(d / 8), 0, st>>>(gU, cwf, f.flags, gX0, (int)B, (int)T,
                                                                           (int)d, s.C);
  k_conv_grad_weight_parts<<<dim3((unsigned)((d + 255) / 256), kConvParts), 256, 0, st>>>(
      gU, static_cast<const __nv_bfloat16*>(X0), f.flags, cpart, (int)B, (int)T, (int)d, s.C);
  k_conv_grad_weight_reduce<<<(unsigned)((d * kTaps + 255) / 256), 256, 0, st>>>(cpart, gcw, (int)d);
  return cudaGetLastError();
}


}  // namespace bwd
}  // namespace ipttt
