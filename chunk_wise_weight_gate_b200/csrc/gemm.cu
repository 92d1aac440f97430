// General bf16 tensor-core GEMM for the backward of the layer (see gemm.h).
//
// One persistent, warp-specialised kernel, one CTA per SM: warp 0 issues TMA
// loads into a ring of four 48 KB stages (a 128 x 64 A tile and a 64 x 256 B
// tile), one thread of warp 1 issues tcgen05.mma (M = 128, N = 256, K = 16) into
// one of two fp32 accumulators of 256 TMEM columns, and eight epilogue warps
// drain the other accumulator (32 rows x 128 columns each) into fp32 or bf16.
// Tiles are handed out statically (tile = block + j * grid), and in the chunk
// modes ordered with the row tiles fastest, so the tiles that read one B slice
// of a chunk run at the same time.  Every wait is bounded and reports
// IPTTT_ERR_TIMEOUT in the status word.
#include "gemm.h"

#include <cuda_bf16.h>

#include <algorithm>

#include "tc.cuh"

namespace ipttt {
namespace gemm {

using namespace ipttt::tc;

namespace {

constexpr int TM = 128, TN = 256, TK = 64, STAGES = 4;
constexpr int A_BYTES = TM * TK * 2;   // 16 KB
constexpr int B_BYTES = TN * TK * 2;   // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int ACC_COLS = 256;
constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 256;
static_assert(SMEM <= 232448, "gemm kernel exceeds shared memory");

struct Tile {
  int b, chunk;  // batch row and chunk (chunk modes)
  int m0, n0;    // tile origin in the output's m and n
  int t0;        // chunk modes: first token of the chunk
  int mrows;     // rows of the output the tile may write (m < mrows)
  int nk;        // K blocks of 64
  int z_b;       // outer coordinate of the B operand
};

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int num_tiles(const Args& a) {
  const int nt = cdiv(a.N, TN);
  if (a.mode == GM_PLAIN) return cdiv(a.M, TM) * nt;
  const int mt = a.mode == GM_CHUNK_ROWS ? cdiv(a.C, TM) : cdiv(a.M, TM);
  return a.nchunks * a.B * nt * mt;
}

__device__ __forceinline__ void decode(const Args& a, int tile, Tile& t) {
  const int nt = cdiv(a.N, TN);
  if (a.mode == GM_PLAIN) {
    const int mt = cdiv(a.M, TM);
    t.b = 0;
    t.chunk = 0;
    t.m0 = (tile % mt) * TM;
    t.n0 = (tile / mt) * TN;
    t.t0 = 0;
    t.mrows = a.M;
    t.nk = cdiv(a.K, TK);
    t.z_b = 0;
    return;
  }
  const int mt = a.mode == GM_CHUNK_ROWS ? cdiv(a.C, TM) : cdiv(a.M, TM);
  const int per_b = nt * mt;
  const int per_chunk = a.B * per_b;
  t.chunk = a.chunk0 + tile / per_chunk;
  const int r = tile % per_chunk;
  t.b = r / per_b;
  const int q = r % per_b;
  t.m0 = (q % mt) * TM;  // row tiles fastest
  t.n0 = (q / mt) * TN;
  t.t0 = t.chunk * a.C;
  const int len = min(a.C, a.T - t.t0);  // tokens of the chunk
  if (a.mode == GM_CHUNK_ROWS) {
    t.mrows = len;
    t.nk = cdiv(a.K, TK);
    t.z_b = (t.chunk % a.nslots) * a.B + t.b;
  } else {
    t.mrows = a.M;
    t.nk = cdiv(len, TK);
    t.z_b = t.b;
  }
}

// Stage loads for K block kb of tile t.
__device__ __forceinline__ void load_stage(const Args& a, const Tile& t, int kb, uint8_t* sa, uint8_t* sb,
                                           uint64_t* bar) {
  const int k = kb * TK;
  // A: rows m0 .. m0 + 127 by k .. k + 63
  if (a.mode == GM_CHUNK_K) {
    // A(b, t, m), MN-major over the chunk's tokens
    tma_load_3d(sa, &a.amap, bar, t.m0, t.t0 + k, t.b);
    tma_load_3d(sa + A_BYTES / 2, &a.amap, bar, t.m0 + 64, t.t0 + k, t.b);
  } else if (a.a_mn) {
    const int z = a.mode == GM_CHUNK_ROWS ? t.b : 0;
    tma_load_3d(sa, &a.amap, bar, t.m0, k, z);
    tma_load_3d(sa + A_BYTES / 2, &a.amap, bar, t.m0 + 64, k, z);
  } else {
    const int row = a.mode == GM_CHUNK_ROWS ? t.t0 + t.m0 : t.m0;
    const int z = a.mode == GM_CHUNK_ROWS ? t.b : 0;
    tma_load_3d(sa, &a.amap, bar, k, row, z);
  }
  // B: k .. k + 63 by columns n0 .. n0 + 255
  if (a.mode == GM_CHUNK_K) {
#pragma unroll
    for (int q = 0; q < 4; ++q) tma_load_3d(sb + q * (B_BYTES / 4), &a.bmap, bar, t.n0 + 64 * q, t.t0 + k, t.b);
  } else if (a.b_mn) {
#pragma unroll
    for (int q = 0; q < 4; ++q) tma_load_3d(sb + q * (B_BYTES / 4), &a.bmap, bar, t.n0 + 64 * q, k, t.z_b);
  } else {
    tma_load_3d(sb, &a.bmap, bar, k, t.n0, t.z_b);
  }
}

__device__ __forceinline__ bool keep_row(const Args& a, const Tile& t, int m) {
  if (m >= t.mrows) return false;
  if (a.mode != GM_CHUNK_ROWS || a.rows == GR_ALL) return true;
  const ChunkMeta cm = a.meta[(size_t)t.b * a.k + t.chunk];
  const int tok = t.t0 + m;
  return a.rows == GR_LAST ? tok >= cm.last_start : (cm.cont && tok < cm.first_end);
}

__global__ void __launch_bounds__(THREADS, 1) gemm_kernel(const __grid_constant__ Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* counters = reinterpret_cast<uint32_t*>(tmem_slot + 2);  // [0] issued, [1] consumed

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = num_tiles(a);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&acc_full[q], 1);
      mbar_init(&acc_empty[q], EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    counters[0] = counters[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&a.amap);
    prefetch_tmap(&a.bmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * ACC_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
        Tile t;
        decode(a, tile, t);
        for (int kb = 0; kb < t.nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait_or_abort(&empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
          uint8_t* sa = stages + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          load_stage(a, t, kb, sa, sa + A_BYTES, &full[s]);
        }
      }
      if (!ok) { *abort_flag = 1; set_status(a.status, IPTTT_ERR_TIMEOUT); }
      counters[0] = it;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const bool amn = a.mode == GM_CHUNK_K ? true : a.a_mn != 0;
      const bool bmn = a.mode == GM_CHUNK_K ? true : a.b_mn != 0;
      const uint32_t idesc = idesc_bf16(TM, TN, amn, bmn);
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tcount) {
        Tile t;
        decode(a, tile, t);
        const int buf = tcount & 1;
        const uint32_t aph = (tcount >> 1) & 1;
        if (!mbar_wait_or_abort(&acc_empty[buf], aph ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tacc = tmem_base + buf * ACC_COLS;
        for (int kb = 0; kb < t.nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait_or_abort(&full[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int ks = 0; ks < TK / 16; ++ks) {
            // MN-major: 16 K rows of 128 B per step, 64-wide MN blocks 64 rows
            // (8 KB) apart.  K-major: 32 B per step inside the 128-byte rows.
            const uint64_t ad = amn ? sdesc_sw128(a_addr + ks * 2048, TK * 128, 1024)
                                    : sdesc_sw128(a_addr + ks * 32, 16, 1024);
            const uint64_t bd = bmn ? sdesc_sw128(b_addr + ks * 2048, TK * 128, 1024)
                                    : sdesc_sw128(b_addr + ks * 32, 16, 1024);
            mma_bf16(tacc, ad, bd, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[buf]);
      }
      if (!ok) { *abort_flag = 1; set_status(a.status, IPTTT_ERR_TIMEOUT); }
      counters[1] = it;
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = ew >> 2;      // 128-column half of the tile it drains
    const int row = quarter * 32 + lane;
    uint32_t tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
      Tile t;
      decode(a, tile, t);
      const int buf = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      if (!mbar_wait(&acc_full[buf], aph)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * ACC_COLS + ((uint32_t)(quarter * 32) << 16) + 128 * half;
      const int m = t.m0 + row;
      const bool keep = keep_row(a, t, m);
      const float s = a.scale ? (a.mode == GM_PLAIN ? a.scale[0] : a.scale[(size_t)t.b * a.k + t.chunk]) : 1.0f;
      long long base;
      if (a.mode == GM_PLAIN) base = (long long)m * a.ldo;
      else if (a.mode == GM_CHUNK_ROWS) base = (long long)t.b * a.osz + (long long)(t.t0 + m) * a.ldo;
      else base = ((long long)t.chunk * a.B + t.b) * a.osz + (long long)m * a.ldo;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t r[32];
        tmem_ld32(tacc + 32 * q, r);
        tmem_ld_wait();
        const int n = t.n0 + 128 * half + 32 * q;
        if (!keep || n >= a.N) continue;
        if (a.out_kind == GO_BF16) {
          uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + base + n);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 w;
            __nv_bfloat162 p0 = __floats2bfloat162_rn(s * __uint_as_float(r[8 * e + 0]), s * __uint_as_float(r[8 * e + 1]));
            __nv_bfloat162 p1 = __floats2bfloat162_rn(s * __uint_as_float(r[8 * e + 2]), s * __uint_as_float(r[8 * e + 3]));
            __nv_bfloat162 p2 = __floats2bfloat162_rn(s * __uint_as_float(r[8 * e + 4]), s * __uint_as_float(r[8 * e + 5]));
            __nv_bfloat162 p3 = __floats2bfloat162_rn(s * __uint_as_float(r[8 * e + 6]), s * __uint_as_float(r[8 * e + 7]));
            w.x = *reinterpret_cast<uint32_t*>(&p0);
            w.y = *reinterpret_cast<uint32_t*>(&p1);
            w.z = *reinterpret_cast<uint32_t*>(&p2);
            w.w = *reinterpret_cast<uint32_t*>(&p3);
            o[e] = w;
          }
        } else {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(a.out) + base + n);
          const bool add = a.out_kind == GO_F32_ADD;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float4 v = make_float4(s * __uint_as_float(r[4 * e + 0]), s * __uint_as_float(r[4 * e + 1]),
                                   s * __uint_as_float(r[4 * e + 2]), s * __uint_as_float(r[4 * e + 3]));
            if (add) {
              const float4 old = o[e];
              v.x += old.x;
              v.y += old.y;
              v.z += old.z;
              v.w += old.w;
            }
            o[e] = v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
    if (!ok) { *abort_flag = 1; set_status(a.status, IPTTT_ERR_TIMEOUT); }
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // Wait (bounded) for copies that were issued but never consumed, so no TMA
    // write lands in shared memory after the block has exited.
    for (uint32_t it = counters[1]; it < counters[0]; ++it) mbar_wait(&full[it % STAGES], (it / STAGES) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * ACC_COLS);
  }
}

}  // namespace

cudaError_t run(const Args& a, int num_sms, cudaStream_t st) {
  if (a.N <= 0 || a.N % 32 != 0 || !a.out) return cudaErrorInvalidValue;
  long long tiles;
  const long long nt = (a.N + TN - 1) / TN;
  if (a.mode == GM_PLAIN) {
    if (a.M <= 0 || a.K <= 0) return cudaErrorInvalidValue;
    tiles = (long long)((a.M + TM - 1) / TM) * nt;
  } else {
    if (a.B <= 0 || a.C <= 0 || a.C % TK != 0 || a.nchunks <= 0 || a.chunk0 < 0 || a.chunk0 + a.nchunks > a.k)
      return cudaErrorInvalidValue;
    if (a.mode == GM_CHUNK_ROWS && (a.K <= 0 || a.nslots <= 0)) return cudaErrorInvalidValue;
    if (a.mode == GM_CHUNK_K && a.M <= 0) return cudaErrorInvalidValue;
    if (a.mode == GM_CHUNK_ROWS && a.rows != GR_ALL && !a.meta) return cudaErrorInvalidValue;
    const long long mt = a.mode == GM_CHUNK_ROWS ? (a.C + TM - 1) / TM : (a.M + TM - 1) / TM;
    tiles = (long long)a.nchunks * a.B * nt * mt;
  }
  if (tiles <= 0 || tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::max(1LL, std::min(tiles, (long long)num_sms));
  gemm_kernel<<<grid, THREADS, SMEM, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gemm
}  // namespace ipttt
