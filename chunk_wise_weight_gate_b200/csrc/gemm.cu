// General bf16 tensor-core GEMM for the backward of the layer (see gemm.h).
//
// One persistent, warp-specialised kernel in two forms:
//   PAIR = true : clusters of two CTAs on neighbouring SMs own 256 x 256 output
//                 tiles; the even CTA issues tcgen05.mma.cta_group::2 (M = 256,
//                 N = 256, K = 16), each CTA loads its 128 A rows and its half
//                 (128 columns) of B into its own shared memory, with completion
//                 counted on the even CTA's barrier (no multicast loads); MMA
//                 completions go to both CTAs; each CTA drains its 128 rows.
//                 128 K per stage (8 MMAs, three 64 KB stages per CTA): 64 bytes
//                 per MMA clock per SM, and the per-stage barrier round trip paid
//                 once per 1024 MMA clocks.
//   PAIR = false: one CTA per 128 x 256 tile, 64 K per stage (four 48 KB
//                 stages), for the per-chunk-rows form when the chunk length is
//                 not a multiple of 256, for small M, per-chunk K of chunks that
//                 are not a multiple of 128 tokens, and where clusters of two
//                 cannot run.
// Warp 0 issues TMA loads into the ring of stages, one thread of warp 1 issues the
// MMAs into one of two fp32 accumulators of 256 TMEM columns, and eight epilogue
// warps drain the other (32 rows x 128 columns each) into fp32 or bf16.  Tiles are
// handed out statically (tile = worker + j * workers), and in the chunk forms
// ordered with the row tiles fastest, so the tiles that read one B slice of a
// chunk run at the same time.  Every wait is bounded and reports
// IPTTT_ERR_TIMEOUT in the status word.
#include "gemm.h"

#include <cuda_bf16.h>

#include <algorithm>

#include "tc.cuh"
#include "tc_kernels.h"

namespace ipttt {
namespace gemm {

using namespace ipttt::tc;

namespace {

constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int ACC_COLS = 256;

template <bool PAIR> struct Cfg {
  static constexpr int TK = PAIR ? 128 : 64;       // K per stage
  static constexpr int TM = PAIR ? 256 : 128;      // output rows of a tile
  static constexpr int BCOLS = PAIR ? 128 : 256;   // B columns one CTA loads
  static constexpr int A_BYTES = 128 * TK * 2;     // this CTA's 128 A rows
  static constexpr int B_BYTES = BCOLS * TK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = PAIR ? 3 : 4;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 256;
};

// The kernel's parameters: the two tensor maps (64-byte aligned, first) and the call.
struct KArgs {
  CUtensorMap amap, bmap;
  Args a;
};
static_assert(Cfg<true>::SMEM <= 232448 && Cfg<false>::SMEM <= 232448, "gemm kernel exceeds shared memory");

struct Tile {
  int b, chunk;  // batch row and chunk (chunk modes)
  int m0, n0;    // tile origin in the output's m and n
  int t0;        // chunk modes: first token of the chunk
  int mrows;     // rows of the output the tile may write (m < mrows)
  int nk;        // K blocks of the tile
  int kb0;       // its first K block
  int slice;     // PLAIN with split K: the slice of K (output matrix)
  int z_b;       // outer coordinate of the B operand
};

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

template <bool PAIR>
__device__ __forceinline__ int num_tiles(const Args& a) {
  constexpr int TM = Cfg<PAIR>::TM;
  const int nt = cdiv(a.N, 256);
  if (a.mode == GM_PLAIN) return cdiv(a.M, TM) * nt * max(1, a.ksplit);
  const int mt = a.mode == GM_CHUNK_ROWS ? cdiv(a.C, TM) : cdiv(a.M, TM);
  return a.nchunks * a.B * nt * mt;
}

template <bool PAIR>
__device__ __forceinline__ void decode(const Args& a, int tile, Tile& t) {
  constexpr int TM = Cfg<PAIR>::TM;
  const int nt = cdiv(a.N, 256);
  if (a.mode == GM_PLAIN) {
    const int mt = cdiv(a.M, TM);
    const int per_slice = mt * nt;
    const int ks = max(1, a.ksplit);
    const int nk_all = cdiv(a.K, Cfg<PAIR>::TK);
    t.slice = tile / per_slice;
    const int r = tile % per_slice;
    t.b = 0;
    t.chunk = 0;
    t.m0 = (r % mt) * TM;
    t.n0 = (r / mt) * 256;
    t.t0 = 0;
    t.mrows = a.M;
    t.kb0 = (int)((long long)nk_all * t.slice / ks);
    t.nk = (int)((long long)nk_all * (t.slice + 1) / ks) - t.kb0;
    t.z_b = 0;
    return;
  }
  t.slice = 0;
  t.kb0 = 0;
  const int mt = a.mode == GM_CHUNK_ROWS ? cdiv(a.C, TM) : cdiv(a.M, TM);
  const int per_b = nt * mt;
  const int per_chunk = a.B * per_b;
  t.chunk = a.chunk0 + tile / per_chunk;
  const int r = tile % per_chunk;
  t.b = r / per_b;
  const int q = r % per_b;
  t.m0 = (q % mt) * TM;  // row tiles fastest
  t.n0 = (q / mt) * 256;
  t.t0 = t.chunk * a.C;
  const int len = min(a.C, a.T - t.t0);  // tokens of the chunk
  if (a.mode == GM_CHUNK_ROWS) {
    t.mrows = len;
    t.nk = cdiv(a.K, Cfg<PAIR>::TK);
    t.z_b = (t.chunk % a.nslots) * a.B + t.b;
  } else {
    t.mrows = a.M;
    t.nk = cdiv(len, Cfg<PAIR>::TK);
    t.z_b = t.b;
  }
}

// One box into this CTA's shared memory; in the pair form completion is counted
// on the even CTA's barrier (its cluster address `bar_c`).
template <bool PAIR>
__device__ __forceinline__ void load_box(void* dst, const CUtensorMap* m, uint64_t* bar, uint32_t bar_c, int x, int y,
                                         int z) {
  if constexpr (PAIR) tma_load_3d_pair(dst, m, bar_c, x, y, z);
  else tma_load_3d(dst, m, bar, x, y, z);
}

// Stage loads of this CTA (rank r) for K block kb of tile t.  Boxes are 64
// elements wide: a K-major operand takes TK / 64 boxes of 128 rows side by side in
// K; an MN-major one takes its 128 (A) or BCOLS (B) columns as 64-wide boxes of TK
// K rows.
template <bool PAIR>
__device__ __forceinline__ void load_stage(const KArgs& ka, const Tile& t, int kb, int r, uint8_t* sa, uint8_t* sb,
                                           uint64_t* bar, uint32_t bar_c) {
  using Cf = Cfg<PAIR>;
  constexpr int TK = Cf::TK, BCOLS = Cf::BCOLS;
  const Args& a = ka.a;
  const int k = (t.kb0 + kb) * TK;
  const int m0 = t.m0 + 128 * r;       // this CTA's A rows
  const int n0 = t.n0 + BCOLS * r;     // this CTA's B columns
  if (a.mode == GM_CHUNK_K || a.a_mn) {
    const int y = a.mode == GM_CHUNK_K ? t.t0 + k : k;
    const int z = a.mode == GM_PLAIN ? 0 : t.b;
#pragma unroll
    for (int q = 0; q < 2; ++q) load_box<PAIR>(sa + q * (64 * TK * 2), &ka.amap, bar, bar_c, m0 + 64 * q, y, z);
  } else {
    const int row = a.mode == GM_CHUNK_ROWS ? t.t0 + m0 : m0;
    const int z = a.mode == GM_CHUNK_ROWS ? t.b : 0;
#pragma unroll
    for (int q = 0; q < TK / 64; ++q) load_box<PAIR>(sa + q * (128 * 64 * 2), &ka.amap, bar, bar_c, k + 64 * q, row, z);
  }
  if (a.mode == GM_CHUNK_K || a.b_mn) {
    const int y = a.mode == GM_CHUNK_K ? t.t0 + k : k;
#pragma unroll
    for (int q = 0; q < BCOLS / 64; ++q)
      load_box<PAIR>(sb + q * (64 * TK * 2), &ka.bmap, bar, bar_c, n0 + 64 * q, y, t.z_b);
  } else {
    // BCOLS rows in blocks of 128, each TK / 64 boxes wide in K
#pragma unroll
    for (int h = 0; h < BCOLS / 128; ++h)
#pragma unroll
      for (int q = 0; q < TK / 64; ++q)
        load_box<PAIR>(sb + (q * (BCOLS / 128) + h) * (128 * 64 * 2), &ka.bmap, bar, bar_c, k + 64 * q,
                       n0 + 128 * h, t.z_b);
  }
}

__device__ __forceinline__ bool keep_row(const Args& a, const Tile& t, int m) {
  if (m >= t.mrows) return false;
  if (a.mode != GM_CHUNK_ROWS || a.rows == GR_ALL) return true;
  const ChunkMeta cm = a.meta[(size_t)t.b * a.k + t.chunk];
  const int tok = t.t0 + m;
  return a.rows == GR_LAST ? tok >= cm.last_start : (cm.cont && tok < cm.first_end);
}

template <bool PAIR>
__global__ void __launch_bounds__(THREADS, 1) gemm_kernel(const __grid_constant__ KArgs ka) {
  using Cf = Cfg<PAIR>;
  constexpr int TK = Cf::TK;
  const Args& a = ka.a;
  constexpr int STAGES = Cf::STAGES;
  constexpr int STAGE_BYTES = Cf::STAGE_BYTES;
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
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const int wk = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;      // worker (pair) index
  const int nwk = PAIR ? (int)cluster_count_x() : (int)gridDim.x;
  const int ntiles = num_tiles<PAIR>(a);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&acc_full[q], 1);
      mbar_init(&acc_empty[q], EPI_WARPS * (PAIR ? 2 : 1));
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    counters[0] = counters[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&ka.amap);
    prefetch_tmap(&ka.bmap);
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
      const uint32_t full0 = PAIR ? map_to_rank(smem_u32(full), 0) : 0u;  // the leader's full[0]
      for (int tile = wk; ok && tile < ntiles; tile += nwk) {
        Tile t;
        decode<PAIR>(a, tile, t);
        for (int kb = 0; kb < t.nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait_or_abort(&empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
          uint8_t* sa = stages + s * STAGE_BYTES;
          // the leader's barrier counts both CTAs' bytes
          if (rank == 0) mbar_arrive_expect_tx(&full[s], (PAIR ? 2 : 1) * STAGE_BYTES);
          load_stage<PAIR>(ka, t, kb, (int)rank, sa, sa + Cf::A_BYTES, &full[s], full0 + 8u * s);
        }
      }
      if (!ok) { *abort_flag = 1; set_status(a.status, IPTTT_ERR_TIMEOUT); }
      counters[0] = it;
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const bool amn = a.mode == GM_CHUNK_K ? true : a.a_mn != 0;
      const bool bmn = a.mode == GM_CHUNK_K ? true : a.b_mn != 0;
      const uint32_t idesc = idesc_bf16(Cf::TM, 256, amn, bmn);
      for (int tile = wk; ok && tile < ntiles; tile += nwk, ++tcount) {
        Tile t;
        decode<PAIR>(a, tile, t);
        const int buf = tcount & 1;
        const uint32_t aph = (tcount >> 1) & 1;
        const bool got = PAIR ? mbar_wait_cluster(&acc_empty[buf], aph ^ 1)
                              : mbar_wait_or_abort(&acc_empty[buf], aph ^ 1, abort_flag);
        if (!got || (PAIR && *abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tacc = tmem_base + buf * ACC_COLS;
        for (int kb = 0; kb < t.nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait_or_abort(&full[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + Cf::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < TK / 16; ++ks) {
            // MN-major: 16 K rows of 128 B per step, 64-wide MN blocks TK rows
            // apart.  K-major: 32 B per step inside the 128-byte rows, the next
            // 64-wide K box (128 A rows, BCOLS B rows) after the first.
            const uint64_t ad = amn ? sdesc_sw128(a_addr + ks * 2048, TK * 128, 1024)
                                    : sdesc_sw128(a_addr + (ks / 4) * (128 * 128) + (ks % 4) * 32, 16, 1024);
            const uint64_t bd = bmn ? sdesc_sw128(b_addr + ks * 2048, TK * 128, 1024)
                                    : sdesc_sw128(b_addr + (ks / 4) * (Cf::BCOLS * 128) + (ks % 4) * 32, 16, 1024);
            const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
            if constexpr (PAIR) mma_bf16_pair(tacc, ad, bd, idesc, acc);
            else mma_bf16(tacc, ad, bd, idesc, acc);
          }
          if constexpr (PAIR) mma_commit_pair(&empty[s], 3); else mma_commit(&empty[s]);
        }
        if (ok) {
          if constexpr (PAIR) mma_commit_pair(&acc_full[buf], 3); else mma_commit(&acc_full[buf]);
        }
      }
      if (!ok) { *abort_flag = 1; set_status(a.status, IPTTT_ERR_TIMEOUT); }
      counters[1] = it;
      if constexpr (PAIR) mma_commit_pair(drain, 1); else mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = ew >> 2;      // 128-column half of the tile it drains
    const int row = 128 * (int)rank + quarter * 32 + lane;
    const uint32_t empty0 = PAIR ? map_to_rank(smem_u32(acc_empty), 0) : 0u;  // the leader's acc_empty[0]
    uint32_t tcount = 0;
    bool ok = true;
    for (int tile = wk; tile < ntiles; tile += nwk, ++tcount) {
      Tile t;
      decode<PAIR>(a, tile, t);
      const int buf = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      if (!mbar_wait(&acc_full[buf], aph)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * ACC_COLS + ((uint32_t)(quarter * 32) << 16) + 128 * half;
      const int m = t.m0 + row;
      const bool keep = keep_row(a, t, m);
      const float s = a.scale ? (a.mode == GM_PLAIN ? a.scale[0] : a.scale[(size_t)t.b * a.k + t.chunk]) : 1.0f;
      long long base;
      if (a.mode == GM_PLAIN) base = (long long)t.slice * a.osz + (long long)m * a.ldo;
      else if (a.mode == GM_CHUNK_ROWS) base = (long long)t.b * a.osz + (long long)(t.t0 + m) * a.ldo;
      else base = ((long long)(t.chunk - a.chunk_base) * a.B + t.b) * a.osz + (long long)m * a.ldo;
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
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              __nv_bfloat162 pr = __floats2bfloat162_rn(s * __uint_as_float(r[8 * e + 2 * h]),
                                                        s * __uint_as_float(r[8 * e + 2 * h + 1]));
              wp[h] = *reinterpret_cast<uint32_t*>(&pr);
            }
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
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(empty0 + 8u * buf);
        else mbar_arrive(&acc_empty[buf]);
      }
    }
    if (!ok) { *abort_flag = 1; set_status(a.status, IPTTT_ERR_TIMEOUT); }
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && rank == 0) {
    // Wait (bounded) for copies that were issued but never consumed, so no TMA
    // write lands in shared memory after the block has exited.
    for (uint32_t it = counters[1]; it < counters[0]; ++it) mbar_wait(&full[it % STAGES], (it / STAGES) & 1);
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, 2 * ACC_COLS);
    else tmem_dealloc(tmem_base, 2 * ACC_COLS);
  }
}

// Clusters of two that can be resident at once (0: the pair form cannot run).
int pair_workers(cudaStream_t st) {
  static int cached[64];
  static bool have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (have[dev]) return cached[dev];
  int n = 0;
  constexpr int smem = Cfg<true>::SMEM;
  if (cudaFuncSetAttribute(gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel<true>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached[dev] = n;
  have[dev] = true;
  return n;
}

long long tiles_of(const Args& a, int tm) {
  const long long nt = (a.N + 255) / 256;
  if (a.mode == GM_PLAIN) return (long long)((a.M + tm - 1) / tm) * nt * std::max(1, a.ksplit);
  const long long mt = a.mode == GM_CHUNK_ROWS ? (a.C + tm - 1) / tm : (a.M + tm - 1) / tm;
  return (long long)a.nchunks * a.B * nt * mt;
}

}  // namespace

cudaError_t run(const Args& a, int num_sms, cudaStream_t st) {
  if (a.N <= 0 || a.N % 32 != 0 || !a.out || !a.A.base || !a.Bop.base) return cudaErrorInvalidValue;
  if (a.mode == GM_PLAIN) {
    // every slice holds at least one K block of either form (64 or 128 K)
    if (a.M <= 0 || a.K <= 0 || a.ksplit < 0 || (a.ksplit > 1 && a.ksplit > a.K / 128)) return cudaErrorInvalidValue;
  } else {
    if (a.ksplit > 1) return cudaErrorInvalidValue;
    if (a.B <= 0 || a.C <= 0 || a.C % 64 != 0 || a.nchunks <= 0 || a.chunk0 < 0 || a.chunk0 + a.nchunks > a.k)
      return cudaErrorInvalidValue;
    if (a.mode == GM_CHUNK_ROWS && (a.K <= 0 || a.nslots <= 0)) return cudaErrorInvalidValue;
    if (a.mode == GM_CHUNK_K && a.M <= 0) return cudaErrorInvalidValue;
    if (a.mode == GM_CHUNK_ROWS && a.rows != GR_ALL && !a.meta) return cudaErrorInvalidValue;
  }
  // Pairs where a 256-row tile is not mostly padding: M of at least 256; in the
  // per-chunk-rows form chunks of a multiple of 256 tokens; in the per-chunk-K
  // form chunks of a multiple of the pair's 128 K per stage.
  const int rows = a.mode == GM_CHUNK_ROWS ? a.C : a.M;
  const bool pair = rows >= 256 && (a.mode != GM_CHUNK_ROWS || a.C % 256 == 0) &&
                    (a.mode != GM_CHUNK_K || a.C % 128 == 0);
  const int np = pair ? pair_workers(st) : 0;
  const int tk = np > 0 ? Cfg<true>::TK : Cfg<false>::TK;
  const bool amn = a.mode == GM_CHUNK_K || a.a_mn;
  const bool bmn = a.mode == GM_CHUNK_K || a.b_mn;
  KArgs ka;
  ka.a = a;
  if (!tck::make_map_bf16(&ka.amap, a.A.base, a.A.inner, a.A.rows, a.A.outer, 64, amn ? tk : 128) ||
      !tck::make_map_bf16(&ka.bmap, a.Bop.base, a.Bop.inner, a.Bop.rows, a.Bop.outer, 64, bmn ? tk : 128))
    return cudaErrorInvalidValue;
  if (np > 0) {
    const long long tiles = tiles_of(a, 256);
    if (tiles <= 0 || tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    constexpr int smem = Cfg<true>::SMEM;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(2 * std::max(1LL, std::min(tiles, (long long)np))), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_kernel<true>, ka);
  }
  const long long tiles = tiles_of(a, 128);
  if (tiles <= 0 || tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  constexpr int smem = Cfg<false>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::max(1LL, std::min(tiles, (long long)num_sms));
  gemm_kernel<false><<<grid, THREADS, smem, st>>>(ka);
  return cudaGetLastError();
}

}  // namespace gemm
}  // namespace ipttt
