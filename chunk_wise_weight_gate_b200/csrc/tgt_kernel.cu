// Target GEMM of the LM-aligned target with its masked depthwise conv computed in
// the producer, so U never reaches HBM:
//   U[t,c] = sum_o conv_w[c,o] X0[t+o,c]   (tap o and every later one dropped once
//                                           t+o reaches the chunk end, T, or a
//                                           document start)
//   V      = U Wtarget, rows outside each chunk's last document segment zeroed
// [cloud.tencent.com "榨干MLP的剩余价值", 详细步骤 3: depthwise conv of kernel 5 that
// never looks past the chunk; lijianxiong.blog notes "In-Place Test-Time Training",
// 对齐语言模型的目标函数: V = Conv1D(X0) Wtarget; iplexlaw.co.kr review §6: chunk and
// document boundaries].
//
// Clusters of two CTAs.  A tile is 256 token rows (128 per CTA) by up to 512
// output columns: per K step two M=256 x N=256 pair MMAs (tcgen05.mma.cta_group::2)
// fill the whole TMEM of both CTAs (2 x 256 fp32 columns each).  Per 64-channel K
// stage:
//   warp 8, one thread : TMA of this CTA's half of the tile's Wtarget columns
//                        (64 x 64 MN-major boxes; completion counted on the even
//                        CTA's barrier, no multicast);
//   warp 9, one thread of the even CTA: the MMAs;
//   warps 0-7          : U for this CTA's 128 rows and the stage's 64 channels, read
//                        from X0 in global memory (each thread 8 channels x 16 rows
//                        through a 20-row window), written as bf16 in the 128-byte-
//                        swizzled K-major layout the MMA reads, then made visible to
//                        the tensor cores (proxy fence, release at cluster scope).
//                        Four groups of two warps take the stages in turn; a group
//                        requests its next window right after publishing a stage.
// The conv arithmetic is that of the stand-alone conv kernel (fp32 FMAs in tap
// order, one bf16 rounding), done two channels per instruction (fma.rn.f32x2).
// There is one accumulator, so the MMAs of a tile wait for the previous tile's
// drain; the same warps drain it (and zero the rows outside the last segment)
// after filling the next tile's first stages, so that those are ready when the
// accumulator is released.  Every wait is bounded and reports IPTTT_ERR_TIMEOUT.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "tc.cuh"
#include "tc_kernels.h"

namespace ipttt {
namespace tck {

using namespace ipttt::tc;

namespace {

constexpr int TG_KB = 64;                     // channels per stage
constexpr int TG_STAGES = 4;
constexpr int TG_A_BYTES = 128 * TG_KB * 2;   // U: this CTA's 128 rows
constexpr int TG_BOX_BYTES = 64 * TG_KB * 2;  // one 64-column Wtarget box
constexpr int TG_B_BYTES = 4 * TG_BOX_BYTES;  // 2 accumulators x this CTA's 128 columns
constexpr int TG_STAGE_BYTES = TG_A_BYTES + TG_B_BYTES;
constexpr int TG_EPI_WARPS = 8;
// Three warpgroups: warps 0-7 conv and epilogue, warp 8 TMA, warp 9 MMA, 10-11
// idle.  Twelve warps cap a thread at 168 registers at launch; the third
// warpgroup drops to 56 and the conv/epilogue warpgroups rise to 224 (an exact
// trade: 128 x (168 - 56) = 256 x (224 - 168)), which holds a second X0 window
// in flight.  The launcher checks the compiled register count.
constexpr int TG_THREADS = 384;
constexpr int TG_WARP_TMA = 8, TG_WARP_MMA = 9;
constexpr int TG_REGS_LAUNCH = 168, TG_REGS_LOW = 56, TG_REGS_EPI = 224;
static_assert((TG_THREADS - 32 * TG_EPI_WARPS) * (TG_REGS_LAUNCH - TG_REGS_LOW) ==
                  32 * TG_EPI_WARPS * (TG_REGS_EPI - TG_REGS_LAUNCH),
              "the register trade of the fused target kernel must balance");
constexpr int TG_SMEM = 1024 + TG_STAGES * TG_STAGE_BYTES + 256;
constexpr int TG_TAPS = 5;
// conv producers: TG_GROUPS groups of two warps, group g filling the stages kb = g
// mod TG_GROUPS; a thread computes TG_RUN rows x 8 channels of its 128 rows
constexpr int TG_GROUPS = 4, TG_RUN = 16;
static_assert(TG_GROUPS * 2 == TG_EPI_WARPS && 8 * TG_RUN == 128, "conv producer layout");
static_assert(TG_SMEM <= 232448, "fused target kernel exceeds shared memory");

struct TgJob {
  int b, m0, n0, nacc;
};

__device__ __forceinline__ bool tg_job(const TcParams& p, uint32_t i, int w, int nw, TgJob& j) {
  const long long tile = (long long)w + (long long)i * nw;
  if (tile >= p.n_tiles) return false;
  // column tiles fastest: the tiles running at one time share their X0 rows in L2
  const int tiles_n = (p.d + 511) / 512;
  const int tiles_m = (p.T + 255) / 256;
  const int nt = (int)(tile % tiles_n);
  const long long mm = tile / tiles_n;
  j.b = (int)(mm / tiles_m);
  j.m0 = (int)(mm % tiles_m) * 256;
  j.n0 = nt * 512;
  j.nacc = min(512, p.d - j.n0) / 256;
  return true;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two fp32 values in one 64-bit register pair, for the packed FMA.
__device__ __forceinline__ unsigned long long f2pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// d = a * b + c on both halves, each an IEEE fp32 fma rounded to nearest.
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// bf16x2 word -> the two values as fp32 (exact)
__device__ __forceinline__ unsigned long long bf2_to_f2(uint32_t w) {
  return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Arrival on the even CTA's barrier that publishes this thread's (fenced) shared
// memory writes to the cluster.
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__global__ void __launch_bounds__(TG_THREADS, 1) tgt_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TG_STAGES * TG_STAGE_BYTES);
  uint64_t* full = bars;                   // [STAGES] even CTA: Wtarget bytes + the conv warps
  uint64_t* empty = bars + TG_STAGES;      // [STAGES] MMA -> producers, both CTAs
  uint64_t* acc_full = empty + TG_STAGES;  // MMA -> epilogue, both CTAs
  uint64_t* acc_empty = acc_full + 1;      // even CTA: 8 epilogue warps of each CTA
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* counters = reinterpret_cast<uint32_t*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int wk = (int)cluster_id_x();
  const int nwk = (int)cluster_count_x();
  const int nk = p.d / TG_KB;  // K stages per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < TG_STAGES; ++s) {
      mbar_init(&full[s], 1 + 2 * (TG_EPI_WARPS / TG_GROUPS));  // TMA + the stage group's warps of both CTAs
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * TG_EPI_WARPS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    counters[0] = counters[1] = 0;
    fence_mbar_init();
  }
  if (warp == TG_WARP_TMA && lane == 0) prefetch_tmap(&p.map[0]);
  if (warp == TG_WARP_MMA) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t full0 = map_to_rank(smem_u32(full), 0);  // the even CTA's full[0]

  if (warp < TG_EPI_WARPS) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(TG_REGS_EPI));
    const int ew = warp;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = ew >> 2;      // epilogue: accumulator (256-column half)
    const int erow = quarter * 32 + lane;
    // conv role: stage group (stages kb = grp mod TG_GROUPS), chunk of 8 channels
    // and run of TG_RUN rows of this CTA's 128
    const int grp = ew >> 1;
    const int cj = lane & 7;
    const int rg = (ew & 1) * 4 + (lane >> 3);
    const __nv_bfloat16* X0 = reinterpret_cast<const __nv_bfloat16*>(p.src0);
    const __nv_bfloat16* cw = reinterpret_cast<const __nv_bfloat16*>(p.src1);
    const uint32_t acc_empty0 = map_to_rank(smem_u32(acc_empty), 0);
    bool ok = true;
    uint32_t tcount = 0;

    // Drains the accumulator of tile jp: this warp's 32 rows, 256 columns.
    auto epilogue = [&](const TgJob& jp, uint32_t tc) -> bool {
      if (!mbar_wait(acc_full, tc & 1)) return false;
      tc_fence_after();
      if (half < jp.nacc) {
        const int t = jp.m0 + 128 * (int)rank + erow;
        const bool valid = t < p.T;
        const int chunk = min(t / p.C, p.k - 1);
        const bool keep = valid && t >= p.meta[(size_t)jp.b * p.k + chunk].last_start;
        __nv_bfloat16* vrow =
            reinterpret_cast<__nv_bfloat16*>(p.out0) + ((size_t)jp.b * p.T + t) * p.d + jp.n0 + 256 * half;
        const uint32_t tacc = tmem_base + 256 * half + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          uint32_t r[32];
          tmem_ld32(tacc + c, r);
          tmem_ld_wait();
          if (valid) {
            uint4* d4 = reinterpret_cast<uint4*>(vrow + c);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w[e] = keep ? pack_bf16x2(__uint_as_float(r[8 * q + 2 * e]), __uint_as_float(r[8 * q + 2 * e + 1]))
                            : 0u;
              d4[q] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);
      return true;
    };

    // Taps in use for this thread's rows of tile jj (the same for every stage of the
    // tile), 3 bits per row.
    auto taps_of = [&](const TgJob& jj) -> uint64_t {
      const int t0 = jj.m0 + 128 * (int)rank + rg * TG_RUN;
      const uint8_t* fl = p.flags + (size_t)jj.b * p.T;
      uint64_t packed = 0;
#pragma unroll
      for (int r = 0; r < TG_RUN; ++r) {
        const int t = t0 + r;
        int n = 1;
        if (t < p.T) {
          const int cend = min((t / p.C + 1) * p.C, p.T);
#pragma unroll
          for (int o = 1; o < TG_TAPS; ++o)
            if (n == o && t + o < cend && !fl[t + o]) n = o + 1;
        }
        packed |= (uint64_t)n << (3 * r);
      }
      return packed;
    };
    // The X0 window (8 channels, TG_RUN + 4 rows) of this thread for stage kb of tile jj.
    auto load_window = [&](uint4 (&x)[TG_RUN + 4], const TgJob& jj, int kb) {
      const int t0 = jj.m0 + 128 * (int)rank + rg * TG_RUN;
      const __nv_bfloat16* xrow = X0 + ((size_t)jj.b * p.T + t0) * p.d + kb * TG_KB + cj * 8;
#pragma unroll
      for (int q = 0; q < TG_RUN + 4; ++q)
        x[q] = (t0 + q < p.T) ? *reinterpret_cast<const uint4*>(xrow + (size_t)q * p.d) : make_uint4(0u, 0u, 0u, 0u);
    };

    // This group's stages are kb = grp, grp + TG_GROUPS, ... of every tile (a tile's
    // stage count is a multiple of TG_GROUPS).  The X0 window of the next one is
    // requested right after this stage is published: the loads then have the
    // other groups' stages to arrive in, and are not in flight when the release
    // below orders this thread's memory operations.
    TgJob j, jn, jprev;
    bool have_prev = false;
    uint4 xr[TG_RUN + 4];
    uint64_t ntp_n = 0;
    bool have_j = tg_job(p, 0, wk, nwk, j);
    if (have_j) {
      ntp_n = taps_of(j);
      load_window(xr, j, grp);
    }
    for (uint32_t i = 0; ok && have_j; ++i) {
      const uint64_t ntp = ntp_n;
      const bool have_jn = tg_job(p, i + 1, wk, nwk, jn);
      for (int kb = grp; kb < nk; kb += TG_GROUPS) {
        if (kb >= TG_STAGES && have_prev) {
          // the next tile's first stages are filled: drain the previous tile
          if (!epilogue(jprev, tcount - 1)) { ok = false; break; }
          have_prev = false;
        }
        const uint32_t it = i * (uint32_t)nk + (uint32_t)kb;
        const int s = it % TG_STAGES;
        const uint32_t ph = (it / TG_STAGES) & 1;
        uint4 wr[5];
        const uint4* wsrc = reinterpret_cast<const uint4*>(cw + (size_t)(kb * TG_KB + cj * 8) * TG_TAPS);
#pragma unroll
        for (int q = 0; q < 5; ++q) wr[q] = wsrc[q];
        if (!mbar_wait_or_abort(&empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
        // weights: tap o of channels (2p, 2p+1) as one fp32 pair
        const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(wr);
        unsigned long long wp[TG_TAPS][4];
#pragma unroll
        for (int o = 0; o < TG_TAPS; ++o)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            wp[o][q] = f2pack(__bfloat162float(wb[(2 * q) * TG_TAPS + o]), __bfloat162float(wb[(2 * q + 1) * TG_TAPS + o]));
        uint8_t* sa = stages + s * TG_STAGE_BYTES;
#pragma unroll
        for (int r = 0; r < TG_RUN; ++r) {
          const int nt = (int)((ntp >> (3 * r)) & 7u);
          unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int o = 0; o < TG_TAPS; ++o) {
            if (o < nt) {
              const uint32_t xw[4] = {xr[r + o].x, xr[r + o].y, xr[r + o].z, xr[r + o].w};
#pragma unroll
              for (int q = 0; q < 4; ++q) acc[q] = fma2(wp[o][q], bf2_to_f2(xw[q]), acc[q]);
            }
          }
          uint32_t ow[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float lo, hi;
            f2unpack(acc[q], lo, hi);
            ow[q] = pack_bf16x2(lo, hi);
          }
          const int row = rg * TG_RUN + r;
          *reinterpret_cast<uint4*>(sa + row * 128 + ((cj ^ (row & 7)) << 4)) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_release_cluster(full0 + 8u * s);
        if (kb + TG_GROUPS < nk) {
          load_window(xr, j, kb + TG_GROUPS);
        } else if (have_jn) {
          ntp_n = taps_of(jn);
          load_window(xr, jn, grp);
        }
      }
      if (!ok) break;
      if (have_prev) {  // a tile of at most STAGES stages
        if (!epilogue(jprev, tcount - 1)) { ok = false; break; }
      }
      jprev = j;
      have_prev = true;
      ++tcount;
      j = jn;
      have_j = have_jn;
    }
    if (ok && have_prev && !epilogue(jprev, tcount - 1)) ok = false;
    if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
    } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(TG_REGS_LOW));
    if (warp == TG_WARP_TMA) {
      if (lane == 0) {
        uint32_t it = 0;
        bool ok = true;
        TgJob j;
        for (uint32_t i = 0; ok && tg_job(p, i, wk, nwk, j); ++i) {
          for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % TG_STAGES;
            const uint32_t ph = (it / TG_STAGES) & 1;
            if (!mbar_wait_or_abort(&empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
            uint8_t* sb = stages + s * TG_STAGE_BYTES + TG_A_BYTES;
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * j.nacc * 2 * TG_BOX_BYTES);
            const uint32_t fb = full0 + 8u * s;
            for (int a = 0; a < j.nacc; ++a)
              for (int q = 0; q < 2; ++q)  // Wtarget[k][n], n contiguous: this CTA's columns of accumulator a
                tma_load_3d_pair(sb + (2 * a + q) * TG_BOX_BYTES, &p.map[0], fb,
                                 j.n0 + 256 * a + 128 * (int)rank + 64 * q, kb * TG_KB, 0);
          }
        }
        if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
        counters[0] = it;
      }
    } else if (warp == TG_WARP_MMA) {
      if (lane == 0 && rank == 0) {
        uint32_t it = 0, tcount = 0;
        bool ok = true;
        TgJob j;
        const uint32_t idesc = idesc_bf16(256, 256, false, true);
        for (uint32_t i = 0; ok && tg_job(p, i, wk, nwk, j); ++i, ++tcount) {
          if (!mbar_wait_cluster(acc_empty, (tcount & 1) ^ 1) || *abort_flag) { ok = false; break; }
          tc_fence_after();
          for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = it % TG_STAGES;
            const uint32_t ph = (it / TG_STAGES) & 1;
            if (!mbar_wait_cluster(&full[s], ph) || *abort_flag) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(stages + s * TG_STAGE_BYTES);
            const uint32_t b_addr = a_addr + TG_A_BYTES;
  #pragma unroll
            for (int ks = 0; ks < TG_KB / 16; ++ks) {
              const uint64_t ad = sdesc_sw128(a_addr + ks * 32, 16, 1024);
              const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
              for (int a = 0; a < j.nacc; ++a) {
                // MN-major: 16 K rows of 128 B per step; the two 64-column blocks of
                // this CTA's half are TG_BOX_BYTES apart
                const uint64_t bd = sdesc_sw128(b_addr + a * 2 * TG_BOX_BYTES + ks * 2048, TG_BOX_BYTES, 1024);
                mma_bf16_pair(tmem_base + 256 * a, ad, bd, idesc, acc);
              }
            }
            mma_commit_pair(&empty[s], 3);
          }
          if (!ok) break;
          mma_commit_pair(acc_full, 3);
        }
        if (!ok) { *abort_flag = 1; set_status(p.status, IPTTT_ERR_TIMEOUT); }
        counters[1] = it;
        mma_commit_pair(drain, 1);
        mbar_wait(drain, 0);
      }
    }
  }
  __syncthreads();
  // After a timeout: let this CTA's issued but never consumed loads land before
  // the shared memory goes away (each wait is bounded).
  if (*abort_flag && threadIdx.x == 0 && rank == 0) {
    for (uint32_t it = counters[1]; it < counters[0]; ++it) mbar_wait(&full[it % TG_STAGES], (it / TG_STAGES) & 1);
  }
  tc_fence_before();
  cluster_sync();
  if (warp == TG_WARP_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace

bool fused_target_supported(int d) { return d % 256 == 0; }

int fused_target_workers(cudaStream_t st) {
  static int cached[64];
  static bool have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (have[dev]) return cached[dev];
  int n = 0;
  // The register trade (setmaxnreg) balances only at the launch register count it
  // was written for; a build compiled to another count is not used.
  cudaFuncAttributes fa;
  const bool regs_ok = cudaFuncGetAttributes(&fa, tgt_kernel) == cudaSuccess && fa.numRegs == TG_REGS_LAUNCH;
  if (regs_ok && cudaFuncSetAttribute(tgt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TG_SMEM) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(TG_THREADS, 1, 1);
    cfg.dynamicSmemBytes = TG_SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, tgt_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached[dev] = n;
  have[dev] = true;
  return n;
}

cudaError_t launch_fused_target(const TcParams& p, cudaStream_t st) {
  if (p.n_tiles <= 0) return cudaSuccess;
  const int np = fused_target_workers(st);
  if (np <= 0) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * std::max(1, std::min(p.n_tiles, np)), 1, 1);
  cfg.blockDim = dim3(TG_THREADS, 1, 1);
  cfg.dynamicSmemBytes = TG_SMEM;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tgt_kernel, p);
}

}  // namespace tck
}  // namespace ipttt
