// C ABI of libipttt (declared in include/ipttt.h): argument checks, workspace
// carve-up, and the order of kernel launches for one In-Place TTT MLP layer.
//
// Launch order (bf16 path), all on the caller's stream:
//   metadata, masked conv U -> Z = SiLU(H Wg^T)*(H Wu^T) -> V = U Wt (last-segment
//   rows) -> Gram partials -> alpha and the pre-scale of V -> per group of chunks:
//   the state updates (S_i -> S_{i+1}, bf16 snapshots) and one launch of the
//   group's apply tiles (reads S_i).
// The chunk order follows lijianxiong.blog notes "In-Place Test-Time Training",
// 方法 (apply with the current fast weight, then update) and iplexlaw.co.kr review
// §3 (a chunk's output always comes from the pre-update state).
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "aux_kernels.h"
#include "common.cuh"
#include "tc_kernels.h"
#include "gemm.h"

namespace ipttt {

__device__ int g_status_word = 0;

ipttt_status cuda_status(cudaError_t e) { return e == cudaSuccess ? IPTTT_OK : IPTTT_ERR_CUDA; }

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int* status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

ipttt_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return IPTTT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    if (cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return IPTTT_ERR_CUDA;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) return IPTTT_ERR_CUDA;
    di.status = static_cast<int*>(addr);
    di.ready = true;
  }
  *out = &di;
  return IPTTT_OK;
}

// ---------------------------------------------------------------- profiling
constexpr int kPhases = 6;
enum Phase { PH_PREP = 0, PH_GATEUP = 1, PH_TARGET = 2, PH_GRAM = 3, PH_APPLY = 4, PH_UPDATE = 5 };

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_profile_on{0};

struct Profiler {
  std::mutex mu;
  std::vector<cudaEvent_t> pool;
  struct Pending {
    cudaEvent_t a, b;
    int phase;
    uint64_t launches;
  };
  std::vector<Pending> pending;
  double ms[kPhases] = {0};
  uint64_t launches[kPhases] = {0};

  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};
Profiler g_prof;

// Brackets one phase of a call: records an event now and one when finished.
struct PhaseScope {
  cudaStream_t st;
  int phase;
  uint64_t start_count;
  cudaEvent_t a = nullptr;
  PhaseScope(cudaStream_t s, int ph) : st(s), phase(ph), start_count(g_launches.load()) {
    if (g_profile_on.load()) {
      std::lock_guard<std::mutex> lk(g_prof.mu);
      a = g_prof.get();
      if (a) cudaEventRecord(a, st);
    }
  }
  ~PhaseScope() {
    if (!a) return;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    cudaEvent_t b = g_prof.get();
    if (!b) return;
    cudaEventRecord(b, st);
    g_prof.pending.push_back({a, b, phase, g_launches.load() - start_count});
  }
};

inline void counted(long long n) { g_launches.fetch_add((uint64_t)n); }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct Layout {
  size_t flags, meta, alpha, partials, Z, U, V, S, snap, raw, dpart, total;
  size_t gmeta, glo, P, E;  // grouped scan: group metadata, per-token group offsets, within-group terms
  bool grouped;
  size_t cp_docs, cp_plan;  // context-parallel calls: local document starts, per-row plan
  int group;  // bf16 path: chunks whose apply tiles share one launch (= snapshot ring slots)
  bool keep_all;  // bf16 forward run for the backward: every chunk's state copy kept, U written
};

// Apply tiles of `group` consecutive chunks share one launch (and the snapshot
// ring has `group` slots).  A launch holds at least kApplyTilesPerLaunch tiles;
// beyond that the group is the smallest one that minimises the apply's waves over
// kWaveCtas CTAs (the SMs of a B200) summed over all launches, within a ring of
// at most kRingBytesMax.
constexpr int kApplyTilesPerLaunch = 1280;
constexpr int kWaveCtas = 148;
constexpr size_t kRingBytesMax = size_t(8) << 30;

// Token rows of an apply or Gram tile: 128, or 64 for chunks that are odd
// multiples of 64 (the MMA still spans 128 rows; the upper 64 are not used).
int tile_rows(const ipttt_params& p) { return p.C % 128 == 0 ? 128 : 64; }

// Token rows of an apply tile: 256 (two M=128 MMAs per B stage) when the chunk
// allows it, else the Gram tile rows.
int apply_rows(const ipttt_params& p) { return p.C % 256 == 0 ? 256 : tile_rows(p); }

int apply_group(const ipttt_params& p) {
  const long long k = (p.T + p.C - 1) / p.C;
  const long long per_chunk = (long long)p.B * (p.C / apply_rows(p)) * (p.d / 128);
  const long long slot_bytes = (long long)p.B * p.d * p.F * 2;
  auto waves = [&](long long g) {
    const long long full = k / g, rest = k % g;
    return full * ((g * per_chunk + kWaveCtas - 1) / kWaveCtas) +
           (rest ? (rest * per_chunk + kWaveCtas - 1) / kWaveCtas : 0);
  };
  long long gmin = (kApplyTilesPerLaunch + per_chunk - 1) / per_chunk;
  gmin = std::max(1LL, std::min(gmin, k));
  const long long gmax = std::max(gmin, std::min(k, (long long)(kRingBytesMax / std::max(1LL, slot_bytes))));
  long long best = gmin, best_waves = waves(gmin);
  for (long long g = gmin + 1; g <= gmax; ++g) {
    const long long w = waves(g);
    if (w < best_waves) {
      best = g;
      best_waves = w;
    }
  }
  return (int)best;
}

bool is_bf16(const ipttt_params& p) { return p.dtype == IPTTT_BF16; }

// Chunks shorter than kGroupTokens (64, 128 or 256 tokens) are scanned
// kGroupTokens at a time: the state is carried, snapshotted and applied per
// group, and the chunks of a group see each other's deltas through the
// within-group term
//   E[t] = sum_{u in an earlier chunk of t's group, in t's document} (z_t . z_u) v'_u
// (v' = alpha eta v on the rows that feed the update).  That equals the
// chunk-by-chunk scan (the apply is linear in the state), with one bf16 state
// snapshot written and read per group instead of per chunk.
constexpr int kGroupTokens = 512;
// The choice depends on the chunk length alone, never on T, so that a call over
// a piece of a sequence (a streamed piece, a host-pipeline piece, a context shard)
// does the same arithmetic as a call over the whole sequence: the grouped scan
// rounds alpha eta v to bf16 before the update, the chunk-by-chunk scan scales
// each fp32 delta instead.  IPTTT_GROUPED_SCAN=0 scans such chunks one by one.
bool grouped_scan(const ipttt_params& p) {
  const char* e = getenv("IPTTT_GROUPED_SCAN");
  if (e && e[0] == '0') return false;
  return is_bf16(p) && p.C < kGroupTokens && kGroupTokens % p.C == 0;
}
}  // namespace

int scan_unit_tokens(const ipttt_params& p) { return grouped_scan(p) ? kGroupTokens : p.C; }

int device_sms() {
  DeviceInfo* di = nullptr;
  return device_info(&di) == IPTTT_OK ? di->num_sms : 0;
}

int* device_status() {
  DeviceInfo* di = nullptr;
  return device_info(&di) == IPTTT_OK ? di->status : nullptr;
}

namespace {

ipttt_params group_params(const ipttt_params& p) {
  ipttt_params g = p;
  g.C = kGroupTokens;
  return g;
}

Shape shape_of(const ipttt_params& p) {
  Shape s;
  s.B = p.B;
  s.T = p.T;
  s.d = p.d;
  s.F = p.F;
  s.C = p.C;
  s.k = (p.T + p.C - 1) / p.C;
  return s;
}

// cp: the layout of the context-parallel calls, whose snapshot ring holds every
// chunk's S_i (k + 1 slots: the apply runs after all the shard's updates) and
// which keep the shard's document starts and per-row plan on the device.
// keep_all: the forward run of the backward, which keeps S_i in slot i for every
// chunk, scans chunk by chunk and writes U.
Layout layout_of(const ipttt_params& p, bool cp = false, bool keep_all = false) {
  const Shape s = shape_of(p);
  const size_t B = s.B, T = s.T, d = s.d, F = s.F, k = s.k;
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.flags = take(B * T);
  L.meta = take(B * k * sizeof(ChunkMeta));
  L.alpha = take(B * k * sizeof(float));
  if (is_bf16(p)) {
    const size_t ct = s.C / tile_rows(p);
    L.partials = take(B * k * (ct * (ct + 1) / 2) * sizeof(float));
    L.Z = take(B * T * F * 2);
    L.U = take(B * T * d * 2);
    L.V = take(B * T * d * 2);
    L.S = take(B * d * F * 4);
    L.keep_all = keep_all;
    // the clip on the accumulated state scales the state chunk by chunk: no grouping
    const bool state_clip = (p.flags & IPTTT_FLAG_STATE_CLIP) != 0;
    L.grouped = !keep_all && !state_clip && grouped_scan(p);
    const size_t kg = (T + kGroupTokens - 1) / kGroupTokens;
    L.group = (cp || keep_all) ? (int)(L.grouped ? kg : s.k) + 1 : apply_group(L.grouped ? group_params(p) : p);
    L.snap = take((size_t)L.group * B * d * F * 2);
    L.raw = L.dpart = 0;
    if (state_clip) {  // each chunk's raw delta in fp32, and the norm's partial sums
      L.raw = take(B * d * F * 4);
      L.dpart = take(B * 148 * 4 * sizeof(double));
    }
    L.gmeta = L.glo = L.P = L.E = 0;
    if (L.grouped) {
      L.gmeta = take(B * kg * sizeof(ChunkMeta));
      L.glo = take(B * T * sizeof(uint16_t));
      L.P = take(B * T * kGroupTokens * 2);
      L.E = take(B * T * d * 2);
    }
  } else {
    L.grouped = false;
    L.gmeta = L.glo = L.P = L.E = 0;
    L.partials = 0;
    L.Z = take(B * T * F * 4);
    L.U = take(B * T * d * 4);
    L.V = take(B * T * d * 4);
    L.S = take(B * d * F * 4);
    L.raw = take(B * d * F * 4);
    L.dpart = take(B * 64 * sizeof(double));
    L.snap = 0;
  }
  L.cp_docs = L.cp_plan = 0;
  if (cp) {
    L.cp_docs = take(B * T * sizeof(int32_t));
    L.cp_plan = take(4 * B * sizeof(int32_t));
  }
  L.total = off;
  return L;
}

ipttt_status check_params(const ipttt_params* p) {
  if (!p) return IPTTT_ERR_ARG;
  if (p->dtype != IPTTT_F32 && p->dtype != IPTTT_BF16) return IPTTT_ERR_DTYPE;
  if (p->B <= 0 || p->T <= 0 || p->d <= 0 || p->F <= 0 || p->C <= 0) return IPTTT_ERR_ARG;
  if (!isfinite(p->eta) || isnan(p->clip_thresh)) return IPTTT_ERR_ARG;
  if ((p->flags & ~(IPTTT_FLAG_RESIDUAL | IPTTT_FLAG_STATE_CLIP)) != 0) return IPTTT_ERR_ARG;
  const long long BT = (long long)p->B * p->T;
  if (BT > (1ll << 30) || (long long)p->d * p->F > (1ll << 31) || (long long)p->d * p->d > (1ll << 31) ||
      BT * (long long)p->F > (1ll << 40))
    return IPTTT_ERR_SHAPE;
  if (p->dtype == IPTTT_BF16) {
    if (p->d % 128 != 0 || p->F % 128 != 0 || p->C % 64 != 0 || p->C > 4096) return IPTTT_ERR_UNSUPPORTED;
  }
  return IPTTT_OK;
}

struct Tensors {
  const void *H, *X0, *Wg, *Wu, *W0, *cw, *Wt;
  const void *Zin, *Vin;  // ipttt_core
  const int32_t* doc;
  int n_doc;
  void* O;
  float *D, *Sfinal, *alpha;
  void *Zout, *Vout;
  void* deltas;  // keep_all forward: every chunk's V_L^T Z_L, bf16 [k][B][d][F] (for the backward)
};

struct StreamState {
  float* S;
  long long* pos;
  int32_t* cont;
};

// The two context-parallel stages (ipttt_cp_begin / ipttt_cp_finish).
//   begin : the shard's forward up to its state updates, from a zero state, with the
//           first chunk continuing the row's document where plan row_cont says so;
//           the fp32 state (= the shard's aggregate) is the caller's `agg`.
//   finish: S_in from the gathered aggregates, folded into the snapshots of the
//           chunks that continue the incoming document, then the apply of every
//           chunk and the final state.
enum CpStageKind { kCpBegin = 1, kCpFinish = 2 };
struct CpArgs {
  int stage;
  int world, rank;
  const int32_t* plan;     // device [4][B]: row_cont, first_rank, prefix_chunks, keep
  float* agg;              // begin: the state / aggregate [B][d][F] (blocked tiles)
  const float* gathered;   // finish: [world][B][d][F], every rank's aggregate
  float* Sfinal;           // finish: optional row-major S_final [B][d][F]
};

size_t state_bytes(const ipttt_params& p) {
  const size_t B = p.B;
  return align256(B * p.d * (size_t)p.F * 4) + align256(B * 8) + align256(B * 4);
}

StreamState state_of(const ipttt_params& p, void* state) {
  uint8_t* base = static_cast<uint8_t*>(state);
  StreamState s;
  const size_t sbytes = align256((size_t)p.B * p.d * (size_t)p.F * 4);
  s.S = reinterpret_cast<float*>(base);
  s.pos = reinterpret_cast<long long*>(base + sbytes);
  s.cont = reinterpret_cast<int32_t*>(base + sbytes + align256((size_t)p.B * 8));
  return s;
}

// The detail behind the last IPTTT_ERR_CUDA of this thread (ipttt_last_error_detail).
thread_local char g_err_detail[320];

ipttt_status cuda_fail(const char* step, cudaError_t e) {
  snprintf(g_err_detail, sizeof(g_err_detail), "%s: %s (%s)", step, cudaGetErrorName(e), cudaGetErrorString(e));
  return IPTTT_ERR_CUDA;
}

#define IP_CHECK(expr)                                  \
  do {                                                  \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return cuda_fail(#expr, e_); \
  } while (0)

// Pair (cluster of two) GEMMs can be switched off with IPTTT_GEMM_CTAS=1.
bool pair_gemms_enabled() {
  const char* e = getenv("IPTTT_GEMM_CTAS");
  return !(e && e[0] == '1');
}

// Whether this call scans its chunks in groups: the layout allows it and the
// within-group products can run (CTA pairs).
bool scan_grouped(const Layout& L, cudaStream_t st) {
  return L.grouped && pair_gemms_enabled() && tck::pair_gemm_workers(st) > 0;
}

ipttt_status run_bf16(const ipttt_params& p, const Tensors& t, uint8_t* ws, const Layout& L, StreamState* ss,
                      DeviceInfo* di, cudaStream_t st, const CpArgs* cp = nullptr) {
  using namespace tck;
  const Shape s = shape_of(p);
  uint8_t* flags = ws + L.flags;
  ChunkMeta* meta = reinterpret_cast<ChunkMeta*>(ws + L.meta);
  float* alpha = reinterpret_cast<float*>(ws + L.alpha);
  float* partials = reinterpret_cast<float*>(ws + L.partials);
  void* Z = t.Zin ? const_cast<void*>(t.Zin) : static_cast<void*>(ws + L.Z);
  void* U = ws + L.U;
  void* V = ws + L.V;
  float* S = ss ? ss->S : cp ? cp->agg : reinterpret_cast<float*>(ws + L.S);
  void* snap = ws + L.snap;
  const float tau = (p.clip_thresh > 0.0f && isfinite(p.clip_thresh)) ? p.clip_thresh : 0.0f;
  ipttt_status rc_ = IPTTT_OK;
  // A context-parallel finish reuses everything its begin left in the workspace.
  const bool cp_finish = cp && cp->stage == kCpFinish;

  // Gate/up and target GEMMs on CTA pairs (256-row tiles) where the device runs
  // clusters of two, else one CTA per 128-row tile; a conv kernel writes U first.
  const bool pair_gemm = pair_gemms_enabled() && pair_gemm_workers(st) > 0;
  // IPTTT_FUSED_TARGET=1: the target GEMM with the conv in its producer (U never
  // reaches HBM; slower today than the conv kernel and the pair GEMM, whose U round
  // trip costs less than the producer's conv arithmetic recomputed for every
  // 512-column tile).
  const char* fe = getenv("IPTTT_FUSED_TARGET");
  const bool fused_target = pair_gemm && !L.keep_all && fe && fe[0] == '1' && fused_target_supported(s.d) &&
                            fused_target_workers(st) > 0;
  // the grouped scan's within-group products run on CTA pairs
  const bool grouped = scan_grouped(L, st);
  Shape gs = s;
  gs.C = kGroupTokens;
  gs.k = (s.T + kGroupTokens - 1) / kGroupTokens;
  const Shape& sq = grouped ? gs : s;  // the chunking of the scan
  ChunkMeta* gmeta = grouped ? reinterpret_cast<ChunkMeta*>(ws + L.gmeta) : meta;
  uint16_t* glo = reinterpret_cast<uint16_t*>(ws + L.glo);
  void* Pw = ws + L.P;
  void* Ew = ws + L.E;
  if (!cp_finish) {
    PhaseScope ph(st, PH_PREP);
    IP_CHECK(aux::build_meta(flags, meta, s, t.doc, t.n_doc, ss ? ss->cont : cp ? cp->plan : nullptr, di->status,
                             st));
    counted(3);
    if (grouped) {
      IP_CHECK(aux::group_meta(flags, gmeta, glo, gs, st));
      counted(2);
    }
    if (t.Zin) {
      IP_CHECK(aux::mask_last_segment(IPTTT_BF16, t.Vin, V, meta, s, st));
      counted(1);
    } else if (!fused_target) {
      IP_CHECK(aux::conv_target(IPTTT_BF16, t.X0, t.cw, flags, U, s, st));
      counted(1);
    }
  }

  TcParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.B = s.B;
  tp.T = s.T;
  tp.d = s.d;
  tp.F = s.F;
  tp.C = s.C;
  tp.k = s.k;
  tp.tr = tile_rows(p);
  tp.ct = s.C / tp.tr;
  tp.npairs = tp.ct * (tp.ct + 1) / 2;
  tp.eta = p.eta;
  tp.meta = meta;
  tp.alpha = alpha;
  tp.status = di->status;

  const int zv_fam = pair_gemm ? FAM_ZV2 : FAM_ZV;
  const int zv_rows = pair_gemm ? 256 : 128;
  if (!t.Zin && !cp_finish) {
    PhaseScope ph(st, PH_GATEUP);
    TcParams g = tp;
    g.kind = kind_gateup();
    if (!make_map_bf16(&g.map[0], t.H, s.d, s.T, s.B, 64, 128) ||
        !make_map_bf16(&g.map[1], t.Wg, s.d, s.F, 1, 64, 128) ||
        !make_map_bf16(&g.map[2], t.Wu, s.d, s.F, 1, 64, 128))
      return cuda_fail("tensor maps of the gate/up GEMM", cudaErrorInvalidValue);
    g.out0 = Z;
    g.n_tiles = s.B * ((s.T + zv_rows - 1) / zv_rows) * (s.F / 128);
    IP_CHECK(launch_tc(zv_fam, g, di->num_sms, st));
    counted(1);
  }
  if (!t.Zin && !cp_finish && fused_target) {
    PhaseScope ph(st, PH_TARGET);
    TcParams v = tp;
    if (!make_map_bf16(&v.map[0], t.Wt, s.d, s.d, 1, 64, 64))
      return cuda_fail("tensor map of the fused target GEMM", cudaErrorInvalidValue);
    v.src0 = t.X0;
    v.src1 = t.cw;
    v.flags = flags;
    v.out0 = V;
    v.n_tiles = s.B * ((s.T + 255) / 256) * ((s.d + 511) / 512);
    IP_CHECK(launch_fused_target(v, st));
    counted(1);
  } else if (!t.Zin && !cp_finish) {
    PhaseScope ph(st, PH_TARGET);
    TcParams v = tp;
    v.kind = kind_vhat();
    if (!make_map_bf16(&v.map[0], U, s.d, s.T, s.B, 64, 128) ||
        !make_map_bf16(&v.map[1], t.Wt, s.d, s.d, 1, 64, pair_gemm ? 128 : 64))
      return cuda_fail("tensor maps of the target GEMM", cudaErrorInvalidValue);
    v.out0 = V;
    v.vn = s.d % 256 == 0 ? 256 : 128;
    v.n_tiles = s.B * ((s.T + zv_rows - 1) / zv_rows) * (s.d / v.vn);
    IP_CHECK(launch_tc(zv_fam, v, di->num_sms, st));
    counted(1);
  }
  if (t.Zout) IP_CHECK(cudaMemcpyAsync(t.Zout, Z, (size_t)s.B * s.T * s.F * 2, cudaMemcpyDeviceToDevice, st));
  if (t.Vout) IP_CHECK(cudaMemcpyAsync(t.Vout, V, (size_t)s.B * s.T * s.d * 2, cudaMemcpyDeviceToDevice, st));

  // The clip on the accumulated state takes its factors from the state itself, chunk
  // by chunk in the scan, so it needs no Gram pass.
  const bool state_clip = (p.flags & IPTTT_FLAG_STATE_CLIP) != 0;
  if (!cp_finish && !state_clip) {
    PhaseScope ph(st, PH_GRAM);
    TcParams g = tp;
    // On CTA pairs: 256 x 256 token-block pairs, two partials (one per CTA) each.
    const bool gram2 = pair_gemm && s.C % 256 == 0;
    if (gram2) {
      g.tr = 256;
      g.ct = s.C / 256;
      g.npairs = g.ct * (g.ct + 1) / 2;
    }
    if (!make_map_bf16(&g.map[0], Z, s.F, s.T, s.B, 64, gram2 ? 128 : tp.tr) ||
        !make_map_bf16(&g.map[1], V, s.d, s.T, s.B, 64, gram2 ? 128 : tp.tr))
      return cuda_fail("tensor maps of the Gram pass", cudaErrorInvalidValue);
    g.partials = partials;
    g.n_tiles = s.B * s.k * g.npairs;
    IP_CHECK(launch_tc(gram2 ? FAM_GRAM2 : FAM_GRAM, g, di->num_sms, st));
    IP_CHECK(aux::alpha_from_partials(partials, alpha, s.B * s.k, gram2 ? 2 * g.npairs : tp.npairs, p.eta, tau,
                                      st));
    if (grouped) {
      // a group's update sums several chunks' V^T Z in one accumulator, and the
      // within-group term uses alpha eta v: fold alpha eta into V's rows
      IP_CHECK(aux::prescale_target(V, alpha, s, p.eta, st));
      counted(1);
    }
    counted(2);
  }
  if (grouped && !cp_finish) {
    // within-group term: P = masked Z Z^T per group (256 x 256 blocks on and below
    // the diagonal), then E = P V'
    PhaseScope ph(st, PH_APPLY);
    TcParams z = tp;
    if (!make_map_bf16(&z.map[0], Z, s.F, s.T, s.B, 64, 128))
      return cuda_fail("tensor map of the within-group products", cudaErrorInvalidValue);
    z.glo = glo;
    z.cs = s.C;
    z.gl = kGroupTokens;
    z.out0 = Pw;
    constexpr int nb = kGroupTokens / 256;
    z.n_tiles = s.B * gs.k * (nb * (nb + 1) / 2);
    IP_CHECK(launch_tc(FAM_PZ, z, di->num_sms, st));
    TcParams e = tp;
    e.kind = kind_intra();
    e.gl = kGroupTokens;
    e.vn = s.d % 256 == 0 ? 256 : 128;
    if (!make_map_bf16(&e.map[0], Pw, kGroupTokens, s.T, s.B, 64, 128) ||
        !make_map_bf16(&e.map[1], V, s.d, s.T, s.B, 64, 128))
      return cuda_fail("tensor maps of the within-group term", cudaErrorInvalidValue);
    e.out0 = Ew;
    e.n_tiles = s.B * ((s.T + 255) / 256) * (s.d / e.vn);
    IP_CHECK(launch_tc(FAM_ZV2, e, di->num_sms, st));
    counted(2);
  }
  if (t.alpha && !state_clip)
    IP_CHECK(cudaMemcpyAsync(t.alpha, alpha, (size_t)s.B * s.k * 4, cudaMemcpyDeviceToDevice, st));

  // A context-parallel shard starts from a zero state: S_0 (snapshot slot 0) and
  // the fp32 state are cleared; the incoming state is added in the finish.
  if (cp && !cp_finish) {
    IP_CHECK(cudaMemsetAsync(S, 0, (size_t)s.B * s.d * s.F * 4, st));
    IP_CHECK(cudaMemsetAsync(snap, 0, (size_t)s.B * s.d * s.F * 2, st));
  }
  // A streaming piece that continues a row starts from the carried state S.
  if (ss) {
    PhaseScope ph(st, PH_UPDATE);
    IP_CHECK(aux::state_snapshot(S, snap, s, st));
    counted(1);
  }

  // The scan.  S_i (bf16 snapshot) lives in ring slot i % G.  For each group of G
  // chunks [a, b): state updates of chunks a .. b-2 (each writes S_{j+1}), then
  // one launch with the apply tiles of chunks a .. b-1 (they read S_a .. S_{b-1}),
  // then the update of chunk b-1 (writes S_b into the slot S_a has left).
  const int G = L.group;
  TcParams sc = tp;
  if (grouped) {
    sc.C = gs.C;
    sc.k = gs.k;
    sc.tr = tile_rows(group_params(p));
    sc.meta = gmeta;
    sc.upd_kb = update_tokens_per_stage(s.C);  // a stage never spans two chunks of the group
    sc.intra = Ew;
  } else {
    sc.upd_scale = 1;  // the update multiplies each chunk's delta by alpha eta
  }
  const int arows = grouped ? apply_rows(group_params(p)) : apply_rows(p);
  const int apply_fam = arows == 256 ? FAM_APPLY256 : FAM_APPLY;
  if (!make_map_bf16(&sc.map[0], Z, s.F, s.T, s.B, 64, arows == 256 ? 128 : sc.tr) ||
      (t.W0 && !make_map_bf16(&sc.map[1], t.W0, s.F, s.d, 1, 64, 128)) ||  // no W0: a context-parallel begin
      !make_map_bf16(&sc.map[2], snap, s.F, s.d, (uint64_t)G * s.B, 64, 128) ||
      !make_map_bf16(&sc.map[3], V, s.d, s.T, s.B, 64, update_tokens_per_stage(s.C)) ||
      !make_map_bf16(&sc.map[4], Z, s.F, s.T, s.B, 64, update_tokens_per_stage(s.C)) ||
      !make_map_bf16(&sc.map[5], snap, s.F, s.d, (uint64_t)G * s.B, 64, 32))
    return cuda_fail("tensor maps of the chunk scan", cudaErrorInvalidValue);
  // the forward of the backward also keeps each chunk's raw delta (the update's
  // TMEM product before alpha eta), which the backward would otherwise recompute
  if (L.keep_all && t.deltas && !grouped) {
    if (!make_map_bf16(&sc.map[7], t.deltas, s.F, s.d, (uint64_t)s.k * s.B, 64, 32))
      return cuda_fail("tensor map of the deltas", cudaErrorInvalidValue);
    sc.delta_out = 1;
  }
  // the 256-row apply writes O through shared memory and TMA stores
  if (apply_fam == FAM_APPLY256 && t.O) {
    if (!make_map_bf16(&sc.map[6], t.O, s.d, s.T, s.B, 64, 32))
      return cuda_fail("tensor map of O", cudaErrorInvalidValue);
    sc.o_tma = 1;
  }
  sc.out0 = t.O;
  sc.out1 = t.D;
  sc.resid = (p.flags & IPTTT_FLAG_RESIDUAL) ? t.H : nullptr;
  sc.S = S;
  sc.nslots = G;
  sc.dchunks = 1;
  // (the last chunk's update also writes its delta when the backward wants them)
  const bool need_final = t.Sfinal != nullptr || ss != nullptr || sc.delta_out;
  const int state_tiles = s.B * (s.d / 128) * ((s.F + 255) / 256);  // 128 x 256 tiles
  const int apply_tiles_per_chunk = s.B * (sq.C / arows) * (s.d / 128);
  // State updates of chunks [c0, c1) in one launch: each worker carries its state
  // tiles' fp32 state in registers through all of them and writes S_{c+1}
  // snapshots into slot (c+1) % G.
  auto update = [&](int c0, int c1) -> ipttt_status {
    if (c1 <= c0) return IPTTT_OK;
    PhaseScope ph(st, PH_UPDATE);
    if (state_clip) {
      // Chunk by chunk: the raw delta V_L^T Z_L as a tcgen05 GEMM (fp32 out, V zero
      // outside the last segment), then on the CUDA cores S = c (keep S + eta delta)
      // with c = tau / ||keep S + eta delta||_F when that exceeds tau (fp32 state,
      // row-major), and the bf16 copy of the new state for the apply.
      float* raw = reinterpret_cast<float*>(ws + L.raw);
      double* dpart = reinterpret_cast<double*>(ws + L.dpart);
      for (int c = c0; c < c1; ++c) {
        gemm::Args r{};
        r.mode = gemm::GM_CHUNK_K;
        r.A = {V, (uint64_t)s.d, (uint64_t)s.T, (uint64_t)s.B};
        r.Bop = {Z, (uint64_t)s.F, (uint64_t)s.T, (uint64_t)s.B};
        r.M = s.d;
        r.N = s.F;
        r.B = s.B;
        r.T = s.T;
        r.C = s.C;
        r.k = s.k;
        r.chunk0 = c;
        r.nchunks = 1;
        r.chunk_base = c;
        r.out_kind = gemm::GO_F32;
        r.out = raw;
        r.ldo = s.F;
        r.osz = (long long)s.d * s.F;
        r.status = tp.status;
        IP_CHECK(gemm::run(r, di->num_sms, st));
        void* copy = c + 1 < s.k ? static_cast<uint8_t*>(snap) + (size_t)((c + 1) % G) * s.B * s.d * s.F * 2 : nullptr;
        IP_CHECK(aux::state_clip_step(S, raw, dpart, alpha, meta, s, c, p.eta, tau, copy, st));
        counted(4);
      }
      return IPTTT_OK;
    }
    TcParams q = sc;
    q.chunk = c0;
    q.dchunks = c1 - c0;
    q.apply_chunk0 = 0;
    q.n_tiles = state_tiles;
    IP_CHECK(launch_update(q, di->num_sms, st));
    counted(1);
    return IPTTT_OK;
  };
  if (cp) {
    // begin: every chunk's update in one launch, S_1 .. S_k into slots 1 .. k and
    // the shard's aggregate left in the state.  finish: the incoming state into
    // S_0 .. S_{prefix-1} (and S_final), then the apply of all k chunks.
    if (!cp_finish) return update(0, sq.k);
    {
      PhaseScope ph(st, PH_UPDATE);
      IP_CHECK(aux::cp_combine(cp->gathered, cp->world, cp->rank, cp->plan, snap, G, cp->Sfinal, s, st));
      counted(1);
    }
    PhaseScope ph(st, PH_APPLY);
    TcParams q = sc;
    q.chunk = 0;
    q.dchunks = 1;
    q.apply_chunk0 = 0;
    q.n_tiles = sq.k * apply_tiles_per_chunk;
    IP_CHECK(launch_tc(apply_fam, q, di->num_sms, st));
    counted(1);
    return IPTTT_OK;
  }
  // Group [a, b) of G chunks: the updates of chunks a-1 .. b-2 produce S_a .. S_{b-1}
  // (ring slots a % G .. (b-1) % G, which the previous group's applies have
  // finished reading), then one launch applies chunks a .. b-1.
  for (int a = 0; a < sq.k; a += G) {
    const int b = std::min(a + G, sq.k);
    if ((rc_ = update(std::max(a - 1, 0), b - 1)) != IPTTT_OK) return rc_;
    PhaseScope ph(st, PH_APPLY);
    TcParams q = sc;
    q.chunk = 0;
    q.dchunks = 1;
    q.apply_chunk0 = a;
    q.n_tiles = (b - a) * apply_tiles_per_chunk;
    IP_CHECK(launch_tc(apply_fam, q, di->num_sms, st));
    counted(1);
  }
  if (need_final && (rc_ = update(sq.k - 1, sq.k)) != IPTTT_OK) return rc_;
  if (t.Sfinal) {
    IP_CHECK(aux::state_export(!state_clip, S, t.Sfinal, s, st));
    counted(1);
  }
  if (t.alpha && state_clip)
    IP_CHECK(cudaMemcpyAsync(t.alpha, alpha, (size_t)s.B * s.k * 4, cudaMemcpyDeviceToDevice, st));
  if (ss) {
    IP_CHECK(aux::stream_advance(ss->pos, ss->cont, s.B, s.T, st));
    counted(1);
  }
  return IPTTT_OK;
}

ipttt_status run_f32(const ipttt_params& p, const Tensors& t, uint8_t* ws, const Layout& L, StreamState* ss,
                     DeviceInfo* di, cudaStream_t st) {
  using namespace aux;
  const Shape s = shape_of(p);
  uint8_t* flags = ws + L.flags;
  ChunkMeta* meta = reinterpret_cast<ChunkMeta*>(ws + L.meta);
  float* alpha = reinterpret_cast<float*>(ws + L.alpha);
  const float* Z = t.Zin ? static_cast<const float*>(t.Zin) : reinterpret_cast<float*>(ws + L.Z);
  float* U = reinterpret_cast<float*>(ws + L.U);
  float* V = reinterpret_cast<float*>(ws + L.V);
  float* S = ss ? ss->S : reinterpret_cast<float*>(ws + L.S);
  float* raw = reinterpret_cast<float*>(ws + L.raw);
  double* dpart = reinterpret_cast<double*>(ws + L.dpart);
  const float tau = (p.clip_thresh > 0.0f && isfinite(p.clip_thresh)) ? p.clip_thresh : 0.0f;
  const long long T = s.T, d = s.d, F = s.F;

  IP_CHECK(build_meta(flags, meta, s, t.doc, t.n_doc, ss ? ss->cont : nullptr, di->status, st));
  counted(3 + (t.Zin ? 1 : 3) + 5 * s.k + (ss ? 1 : 0) + (t.Sfinal ? 1 : 0));
  if (!t.Zin) {
    IP_CHECK(conv_target(IPTTT_F32, t.X0, t.cw, flags, U, s, st));
    SimtArgs a{};
    a.M = s.T; a.N = s.F; a.K = s.d;
    a.A = static_cast<const float*>(t.H); a.sam = d; a.sak = 1; a.sab = T * d;
    a.B0 = static_cast<const float*>(t.Wg); a.s0n = d; a.s0k = 1; a.s0b = 0;
    a.B1 = static_cast<const float*>(t.Wu); a.s1n = d; a.s1k = 1; a.s1b = 0;
    a.mode = SM_Z;
    a.out = const_cast<float*>(Z); a.som = F; a.son = 1; a.sob = T * F;
    IP_CHECK(simt_gemm(a, s.B, st));

    SimtArgs v{};
    v.M = s.T; v.N = s.d; v.K = s.d;
    v.A = U; v.sam = d; v.sak = 1; v.sab = T * d;
    v.B0 = static_cast<const float*>(t.Wt); v.s0n = 1; v.s0k = d; v.s0b = 0;
    v.mode = SM_V;
    v.out = V; v.som = d; v.son = 1; v.sob = T * d;
    v.meta = meta; v.k = s.k; v.C = s.C; v.row0 = 0;
    IP_CHECK(simt_gemm(v, s.B, st));
  } else {
    IP_CHECK(mask_last_segment(IPTTT_F32, t.Vin, V, meta, s, st));
  }
  if (t.Zout) IP_CHECK(cudaMemcpyAsync(t.Zout, Z, (size_t)s.B * T * F * 4, cudaMemcpyDeviceToDevice, st));
  if (t.Vout) IP_CHECK(cudaMemcpyAsync(t.Vout, V, (size_t)s.B * T * d * 4, cudaMemcpyDeviceToDevice, st));

  for (int i = 0; i < s.k; ++i) {
    const long long t0 = (long long)i * s.C;
    const int rows = (int)std::min<long long>(s.C, T - t0);
    SimtArgs a{};
    a.M = rows; a.N = s.d; a.K = s.F;
    a.A = Z + t0 * F; a.sam = F; a.sak = 1; a.sab = T * F;
    a.B0 = static_cast<const float*>(t.W0); a.s0n = F; a.s0k = 1; a.s0b = 0;
    a.B1 = S; a.s1n = F; a.s1k = 1; a.s1b = d * F;
    a.mode = SM_APPLY;
    a.out = static_cast<float*>(t.O) + t0 * d; a.som = d; a.son = 1; a.sob = T * d;
    a.out2 = t.D ? t.D + t0 * d : nullptr;
    a.resid = (p.flags & IPTTT_FLAG_RESIDUAL) ? static_cast<const float*>(t.H) + t0 * d : nullptr;
    a.meta = meta; a.k = s.k; a.C = s.C; a.chunk = i; a.row0 = (int)t0;
    IP_CHECK(simt_gemm(a, s.B, st));

    SimtArgs r{};
    r.M = s.d; r.N = s.F; r.K = rows;
    r.A = V + t0 * d; r.sam = 1; r.sak = d; r.sab = T * d;
    r.B0 = Z + t0 * F; r.s0n = 1; r.s0k = F; r.s0b = T * F;
    r.mode = SM_RAW;
    r.out = raw; r.som = F; r.son = 1; r.sob = d * F;
    IP_CHECK(simt_gemm(r, s.B, st));
    if (p.flags & IPTTT_FLAG_STATE_CLIP)
      IP_CHECK(simt_update_state_clipped(S, raw, dpart, alpha, meta, s, i, p.eta, tau, st));
    else
      IP_CHECK(simt_update_state(S, raw, dpart, alpha, meta, s, i, p.eta, tau, st));
  }
  if (t.alpha) IP_CHECK(cudaMemcpyAsync(t.alpha, alpha, (size_t)s.B * s.k * 4, cudaMemcpyDeviceToDevice, st));
  if (t.Sfinal) IP_CHECK(state_export(false, S, t.Sfinal, s, st));
  if (ss) IP_CHECK(stream_advance(ss->pos, ss->cont, s.B, s.T, st));
  return IPTTT_OK;
}

ipttt_status check_tensor(const void* ptr) {
  if (!ptr) return IPTTT_ERR_ARG;
  if (!aligned(ptr, 16)) return IPTTT_ERR_ALIGN;
  return IPTTT_OK;
}

ipttt_status run(const ipttt_params* pp, const Tensors& t, void* workspace, size_t ws_bytes, void* state,
                 void* stream) {
  ipttt_status rc = check_params(pp);
  if (rc != IPTTT_OK) return rc;
  const ipttt_params& p = *pp;
  const bool core = t.Zin != nullptr;
  if (core && (p.flags & IPTTT_FLAG_RESIDUAL)) return IPTTT_ERR_ARG;
  if ((p.flags & IPTTT_FLAG_RESIDUAL) && t.O == t.H) return IPTTT_ERR_ARG;
  const void* must[] = {core ? t.Zin : t.H, core ? t.Vin : t.X0, core ? t.W0 : t.Wg, core ? t.W0 : t.Wu, t.W0,
                        core ? t.W0 : t.cw, core ? t.W0 : t.Wt, t.O};
  for (const void* q : must)
    if ((rc = check_tensor(q)) != IPTTT_OK) return rc;
  const void* optional[] = {t.D, t.Sfinal, t.alpha, t.Zout, t.Vout};
  for (const void* q : optional)
    if (q && !aligned(q, 16)) return IPTTT_ERR_ALIGN;
  if (t.n_doc < 0 || (t.n_doc > 0 && !t.doc)) return IPTTT_ERR_ARG;
  if (t.doc && !aligned(t.doc, 4)) return IPTTT_ERR_ALIGN;
  const Layout L = layout_of(p);
  if (!workspace || ws_bytes < L.total) return IPTTT_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return IPTTT_ERR_ALIGN;
  if (state && !aligned(state, 256)) return IPTTT_ERR_ALIGN;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di)) != IPTTT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  StreamState ss;
  StreamState* ssp = nullptr;
  if (state) {
    // the bf16 state-clip reading keeps its state row-major, the stream state is blocked
    if (is_bf16(p) && (p.flags & IPTTT_FLAG_STATE_CLIP)) return IPTTT_ERR_UNSUPPORTED;
    ss = state_of(p, state);
    ssp = &ss;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  g_err_detail[0] = 0;
  rc = is_bf16(p) ? run_bf16(p, t, ws, L, ssp, di, st) : run_f32(p, t, ws, L, ssp, di, st);
  if (rc == IPTTT_OK && cudaPeekAtLastError() != cudaSuccess) rc = cuda_fail("kernel launch", cudaGetLastError());
  return rc;
}

}  // namespace

ipttt_status validate_params(const ipttt_params* p) { return check_params(p); }

}  // namespace ipttt

using namespace ipttt;

extern "C" {

size_t ipttt_workspace_size(const ipttt_params* p) {
  if (check_params(p) != IPTTT_OK) return 0;
  return layout_of(*p).total;
}

ipttt_status ipttt_forward(const ipttt_params* p, const void* H, const void* X0, const void* Wgate, const void* Wup,
                           const void* Wdown0, const void* conv_w, const void* Wtarget, const int32_t* doc_starts,
                           int32_t n_doc_starts, void* O, void* workspace, size_t workspace_bytes, void* stream) {
  Tensors t{H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, nullptr, nullptr, doc_starts, n_doc_starts, O,
            nullptr, nullptr, nullptr, nullptr, nullptr};
  return run(p, t, workspace, workspace_bytes, nullptr, stream);
}

ipttt_status ipttt_forward_ex(const ipttt_params* p, const void* H, const void* X0, const void* Wgate,
                              const void* Wup, const void* Wdown0, const void* conv_w, const void* Wtarget,
                              const int32_t* doc_starts, int32_t n_doc_starts, void* O, float* D_opt,
                              float* S_final_opt, float* alpha_opt, void* Z_opt, void* V_opt, void* workspace,
                              size_t workspace_bytes, void* stream) {
  Tensors t{H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, nullptr, nullptr, doc_starts, n_doc_starts, O,
            D_opt, S_final_opt, alpha_opt, Z_opt, V_opt};
  return run(p, t, workspace, workspace_bytes, nullptr, stream);
}

ipttt_status ipttt_core(const ipttt_params* p, const void* Z, const void* V, const void* Wdown0,
                        const int32_t* doc_starts, int32_t n_doc_starts, void* O, float* D_opt, float* S_final_opt,
                        float* alpha_opt, void* workspace, size_t workspace_bytes, void* stream) {
  if (!Z || !V) return IPTTT_ERR_ARG;
  Tensors t{nullptr, nullptr, nullptr, nullptr, Wdown0, nullptr, nullptr, Z, V, doc_starts, n_doc_starts, O,
            D_opt, S_final_opt, alpha_opt, nullptr, nullptr};
  return run(p, t, workspace, workspace_bytes, nullptr, stream);
}

size_t ipttt_stream_state_size(const ipttt_params* p) {
  if (check_params(p) != IPTTT_OK) return 0;
  return state_bytes(*p);
}

ipttt_status ipttt_stream_reset(const ipttt_params* p, void* state, void* stream) {
  ipttt_status rc = check_params(p);
  if (rc != IPTTT_OK) return rc;
  if (!state) return IPTTT_ERR_ARG;
  if (!aligned(state, 256)) return IPTTT_ERR_ALIGN;
  return cuda_status(cudaMemsetAsync(state, 0, state_bytes(*p), static_cast<cudaStream_t>(stream)));
}

ipttt_status ipttt_stream_forward(const ipttt_params* p, void* state, const void* H, const void* X0,
                                  const void* Wgate, const void* Wup, const void* Wdown0, const void* conv_w,
                                  const void* Wtarget, const int32_t* doc_starts, int32_t n_doc_starts, void* O,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!state) return IPTTT_ERR_ARG;
  Tensors t{H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, nullptr, nullptr, doc_starts, n_doc_starts, O,
            nullptr, nullptr, nullptr, nullptr, nullptr};
  return run(p, t, workspace, workspace_bytes, state, stream);
}

ipttt_status ipttt_stream_export(const ipttt_params* p, const void* state, float* S_out, void* stream) {
  ipttt_status rc = check_params(p);
  if (rc != IPTTT_OK) return rc;
  if (!state || !S_out) return IPTTT_ERR_ARG;
  if (!aligned(state, 256) || !aligned(S_out, 16)) return IPTTT_ERR_ALIGN;
  const StreamState ss = state_of(*p, const_cast<void*>(state));
  return cuda_status(aux::state_export(is_bf16(*p), ss.S, S_out, shape_of(*p), static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- context parallelism
size_t ipttt_cp_workspace_size(const ipttt_params* p) {
  if (check_params(p) != IPTTT_OK || p->dtype != IPTTT_BF16) return 0;
  return layout_of(*p, true).total;
}

ipttt_status ipttt_cp_plan(const ipttt_params* p, int32_t world, int32_t rank, const int32_t* doc_starts_host,
                           int32_t n_doc_starts, int32_t* local_starts, int32_t* n_local, int32_t* plan) {
  ipttt_status rc = check_params(p);
  if (rc != IPTTT_OK) return rc;
  if (world < 1 || rank < 0 || rank >= world || n_doc_starts < 0 || (n_doc_starts > 0 && !doc_starts_host) ||
      !n_local || !plan)
    return IPTTT_ERR_ARG;
  const long long B = p->B, T = p->T, C = p->C;
  const long long Tg = T * world;
  if (B * Tg > 0x7fffffffLL) return IPTTT_ERR_SHAPE;
  if (world > 1 && T % C != 0) return IPTTT_ERR_SHAPE;
  const long long k = (T + C - 1) / C;
  int32_t* row_cont = plan;
  int32_t* first_rank = plan + B;
  int32_t* prefix = plan + 2 * B;
  int32_t* keep = plan + 3 * B;
  // last[b]: the last rank before this one whose shard of row b holds a start (the
  // row start counts for rank 0); first[b]: this shard's first local start or -1.
  std::vector<long long> last(B, 0), first(B, -1);
  long long prev = -1;
  int32_t m = 0;
  for (int32_t i = 0; i < n_doc_starts; ++i) {
    const long long g = doc_starts_host[i];
    if (g < 0 || g >= B * Tg || g <= prev) return IPTTT_ERR_ARG;
    prev = g;
    const long long b = g / Tg, t = g % Tg, owner = t / T;
    if (owner < rank) last[b] = std::max(last[b], owner);
    if (owner == rank) {
      if (first[b] < 0) first[b] = t - rank * T;
      if (local_starts) local_starts[m] = (int32_t)(b * T + (t - rank * T));
      ++m;
    }
  }
  *n_local = m;
  for (long long b = 0; b < B; ++b) {
    const bool starts_at_0 = rank == 0 || first[b] == 0;
    row_cont[b] = starts_at_0 ? 0 : 1;
    first_rank[b] = rank == 0 ? 0 : (int32_t)last[b];
    prefix[b] = starts_at_0 ? 0 : (int32_t)(first[b] < 0 ? k : first[b] / C + 1);
    keep[b] = (!starts_at_0 && first[b] < 0) ? 1 : 0;
  }
  return IPTTT_OK;
}

}  // extern "C"

namespace ipttt {
namespace {
ipttt_status cp_run(const ipttt_params* p, int32_t world, int32_t rank, const int32_t* doc_starts_host,
                    int32_t n_doc_starts, const Tensors& t, CpArgs cp, void* workspace, size_t workspace_bytes,
                    void* stream) {
  ipttt_status rc = check_params(p);
  if (rc != IPTTT_OK) return rc;
  if (p->dtype != IPTTT_BF16) return IPTTT_ERR_UNSUPPORTED;
  // the shards' aggregates add up only while the update is linear in the state
  if (p->flags & IPTTT_FLAG_STATE_CLIP) return IPTTT_ERR_UNSUPPORTED;
  const Layout L = layout_of(*p, true);
  if (!workspace || workspace_bytes < L.total) return IPTTT_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return IPTTT_ERR_ALIGN;
  int32_t n_local = 0;
  std::vector<int32_t> plan(4 * (size_t)p->B);
  if ((rc = ipttt_cp_plan(p, world, rank, doc_starts_host, n_doc_starts, nullptr, &n_local, plan.data())) !=
      IPTTT_OK)
    return rc;
  std::vector<int32_t> local((size_t)std::max(n_local, 1));
  if ((rc = ipttt_cp_plan(p, world, rank, doc_starts_host, n_doc_starts, local.data(), &n_local, plan.data())) !=
      IPTTT_OK)
    return rc;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di)) != IPTTT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (scan_grouped(L, static_cast<cudaStream_t>(stream))) {
    // the incoming state reaches the groups up to the one holding the shard's
    // first document start (the plan counts chunks)
    for (int32_t b = 0; b < p->B; ++b) {
      int32_t& pre = plan[2 * (size_t)p->B + b];
      if (pre > 0) pre = (int32_t)(((long long)(pre - 1) * p->C) / kGroupTokens + 1);
    }
  }
  int32_t* plan_dev = reinterpret_cast<int32_t*>(ws + L.cp_plan);
  int32_t* docs_dev = reinterpret_cast<int32_t*>(ws + L.cp_docs);
  // pageable sources: the copies have taken the bytes when they return
  IP_CHECK(cudaMemcpyAsync(plan_dev, plan.data(), plan.size() * 4, cudaMemcpyHostToDevice, st));
  if (cp.stage == kCpBegin && n_local > 0)
    IP_CHECK(cudaMemcpyAsync(docs_dev, local.data(), (size_t)n_local * 4, cudaMemcpyHostToDevice, st));
  Tensors tt = t;
  tt.doc = n_local > 0 ? docs_dev : nullptr;
  tt.n_doc = n_local;
  cp.world = world;
  cp.rank = rank;
  cp.plan = plan_dev;
  g_err_detail[0] = 0;
  rc = run_bf16(*p, tt, ws, L, nullptr, di, st, &cp);
  if (rc == IPTTT_OK && cudaPeekAtLastError() != cudaSuccess) rc = cuda_fail("kernel launch", cudaGetLastError());
  return rc;
}
}  // namespace
}  // namespace ipttt

extern "C" {

ipttt_status ipttt_cp_begin(const ipttt_params* p, int32_t world, int32_t rank, const int32_t* doc_starts_host,
                            int32_t n_doc_starts, const void* H, const void* X0, const void* Wgate, const void* Wup,
                            const void* conv_w, const void* Wtarget, float* agg, void* workspace,
                            size_t workspace_bytes, void* stream) {
  ipttt_status rc;
  const void* must[] = {H, X0, Wgate, Wup, conv_w, Wtarget, agg};
  for (const void* q : must)
    if ((rc = check_tensor(q)) != IPTTT_OK) return rc;
  Tensors t{H, X0, Wgate, Wup, nullptr, conv_w, Wtarget, nullptr, nullptr, nullptr, 0, nullptr,
            nullptr, nullptr, nullptr, nullptr, nullptr};
  CpArgs cp{};
  cp.stage = kCpBegin;
  cp.agg = agg;
  return cp_run(p, world, rank, doc_starts_host, n_doc_starts, t, cp, workspace, workspace_bytes, stream);
}

ipttt_status ipttt_cp_finish(const ipttt_params* p, int32_t world, int32_t rank, const int32_t* doc_starts_host,
                             int32_t n_doc_starts, const void* H, const void* Wdown0, const float* gathered,
                             void* O, float* S_final_opt, void* workspace, size_t workspace_bytes, void* stream) {
  ipttt_status rc;
  if (p && (p->flags & IPTTT_FLAG_RESIDUAL) && O == H) return IPTTT_ERR_ARG;
  const void* must[] = {H, Wdown0, gathered, O};
  for (const void* q : must)
    if ((rc = check_tensor(q)) != IPTTT_OK) return rc;
  if (S_final_opt && !aligned(S_final_opt, 16)) return IPTTT_ERR_ALIGN;
  Tensors t{H, nullptr, nullptr, nullptr, Wdown0, nullptr, nullptr, nullptr, nullptr, nullptr, 0, O,
            nullptr, nullptr, nullptr, nullptr, nullptr};
  CpArgs cp{};
  cp.stage = kCpFinish;
  cp.gathered = gathered;
  cp.Sfinal = S_final_opt;
  return cp_run(p, world, rank, doc_starts_host, n_doc_starts, t, cp, workspace, workspace_bytes, stream);
}

ipttt_status ipttt_get_status(void* stream) {
  DeviceInfo* di = nullptr;
  ipttt_status rc = device_info(&di);
  if (rc != IPTTT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return IPTTT_ERR_CUDA;
  if (cudaMemcpyAsync(&v, di->status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return IPTTT_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyAsync(di->status, &zero, sizeof(int), cudaMemcpyHostToDevice, st) != cudaSuccess)
    return IPTTT_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return IPTTT_ERR_CUDA;
  return static_cast<ipttt_status>(v);
}

const char* ipttt_strerror(ipttt_status s) {
  switch (s) {
    case IPTTT_OK: return "ok";
    case IPTTT_ERR_ARG: return "invalid argument";
    case IPTTT_ERR_SHAPE: return "inconsistent or oversized shape";
    case IPTTT_ERR_ALIGN: return "misaligned pointer";
    case IPTTT_ERR_DTYPE: return "unknown dtype";
    case IPTTT_ERR_UNSUPPORTED: return "shape not supported by the bf16 tensor-core path";
    case IPTTT_ERR_CUDA: return "CUDA error";
    case IPTTT_ERR_TIMEOUT: return "a device-side bounded wait gave up";
    case IPTTT_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* ipttt_version(void) { return "0.2.0"; }

// The backward takes the forward's shape rules: any shape in fp32 (CUDA cores),
// the tensor-core shapes in bf16.
// The gradients are those of the per-delta clip; the accumulated-state reading has
// none here.
static ipttt_status backward_params(const ipttt_params* p) {
  const ipttt_status rc = check_params(p);
  if (rc != IPTTT_OK) return rc;
  return (p->flags & IPTTT_FLAG_STATE_CLIP) ? IPTTT_ERR_UNSUPPORTED : IPTTT_OK;
}

// bf16 workspace: the forward's layout with every state copy kept, O of that
// forward, then the backward's own buffers.
struct BwdTcLayout {
  Layout fwd;
  size_t O, tc, total;
};
static BwdTcLayout bwd_tc_layout(const ipttt_params& p) {
  BwdTcLayout L;
  L.fwd = layout_of(p, false, true);
  const Shape s = shape_of(p);
  L.O = align256(L.fwd.total);
  L.tc = L.O + align256((size_t)s.B * s.T * s.d * 2);
  L.total = L.tc + bwd::tc_workspace_bytes(s);
  return L;
}

size_t ipttt_backward_workspace_size(const ipttt_params* p) {
  if (backward_params(p) != IPTTT_OK) return 0;
  if (p->dtype == IPTTT_BF16) return bwd_tc_layout(*p).total;
  return bwd::workspace_bytes(shape_of(*p));
}

ipttt_status ipttt_backward(const ipttt_params* p, const void* H, const void* X0, const void* Wgate, const void* Wup,
                            const void* Wdown0, const void* conv_w, const void* Wtarget, const int32_t* doc_starts,
                            int32_t n_doc_starts, const void* gO, const float* gS_final_opt, float* gH, float* gX0,
                            float* gWgate, float* gWup, float* gWdown0, float* gconv_w, float* gWtarget,
                            void* workspace, size_t workspace_bytes, void* stream) {
  ipttt_status rc = backward_params(p);
  if (rc != IPTTT_OK) return rc;
  if (p->flags != 0) return IPTTT_ERR_ARG;
  const void* must[] = {H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, gO, gH, gX0, gWgate, gWup, gWdown0, gconv_w,
                        gWtarget};
  for (const void* q : must)
    if ((rc = check_tensor(q)) != IPTTT_OK) return rc;
  if (gS_final_opt && !aligned(gS_final_opt, 16)) return IPTTT_ERR_ALIGN;
  if (n_doc_starts < 0 || (n_doc_starts > 0 && !doc_starts)) return IPTTT_ERR_ARG;
  const Shape s = shape_of(*p);
  if (!workspace || workspace_bytes < ipttt_backward_workspace_size(p)) return IPTTT_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return IPTTT_ERR_ALIGN;
  DeviceInfo* di = nullptr;
  if ((rc = device_info(&di)) != IPTTT_OK) return rc;
  const float tau = (p->clip_thresh > 0.0f && isfinite(p->clip_thresh)) ? p->clip_thresh : 0.0f;
  g_err_detail[0] = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->dtype == IPTTT_BF16) {
    // the forward, every state copy kept, then the gradients on the tensor cores
    const BwdTcLayout BL = bwd_tc_layout(*p);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    Tensors t{};
    t.H = H; t.X0 = X0; t.Wg = Wgate; t.Wu = Wup; t.W0 = Wdown0; t.cw = conv_w; t.Wt = Wtarget;
    t.doc = doc_starts;
    t.n_doc = n_doc_starts;
    t.O = ws + BL.O;
    t.deltas = bwd::tc_delta_buffer(ws + BL.tc, s);
    if ((rc = run_bf16(*p, t, ws, BL.fwd, nullptr, di, st)) != IPTTT_OK) return rc;
    bwd::TcForward f;
    f.deltas_ready = !BL.fwd.grouped;
    f.Z = ws + BL.fwd.Z;
    f.U = ws + BL.fwd.U;
    f.V = ws + BL.fwd.V;
    f.snap = ws + BL.fwd.snap;
    f.alpha = reinterpret_cast<const float*>(ws + BL.fwd.alpha);
    f.meta = reinterpret_cast<const ChunkMeta*>(ws + BL.fwd.meta);
    f.flags = ws + BL.fwd.flags;
    f.nslots = BL.fwd.group;
    const cudaError_t e = bwd::run_tc(s, p->eta, tau, f, H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, gO,
                                      gS_final_opt, gH, gX0, gWgate, gWup, gWdown0, gconv_w, gWtarget, ws + BL.tc,
                                      di->status, di->num_sms, st);
    if (e != cudaSuccess) return cuda_fail("backward", e);
    counted(bwd::tc_launches(f.deltas_ready, gS_final_opt != nullptr));
    return IPTTT_OK;
  }
  const cudaError_t e = bwd::run(s, p->dtype, p->eta, tau, H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, doc_starts,
                                 n_doc_starts, gO, gS_final_opt, gH, gX0, gWgate, gWup, gWdown0, gconv_w, gWtarget,
                                 static_cast<uint8_t*>(workspace), di->status, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail("backward", e);
  counted(bwd::launches(s, p->dtype));
  return IPTTT_OK;
}

const char* ipttt_last_error_detail(void) { return g_err_detail; }

}  // extern "C"

// ---------------------------------------------------------------- no-allocation forward
// Scratch for ipttt_forward_noalloc: one static array per device that loads the
// library.  In host code the symbol is only a stand-in for the device array, so
// its device address is looked up (once per device, with that device current)
// and that address is what the kernels get.
static __device__ __align__(256) uint8_t g_noalloc_scratch[IPTTT_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_addr[kMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

ipttt_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return IPTTT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return IPTTT_ERR_CUDA;
    g_noalloc_addr[dev] = addr;
  }
  *out = g_noalloc_addr[dev];
  return IPTTT_OK;
}
}  // namespace

extern "C" {

ipttt_status ipttt_forward_noalloc(const ipttt_params* p, const void* H, const void* X0, const void* Wgate,
                                   const void* Wup, const void* Wdown0, const void* conv_w, const void* Wtarget,
                                   const int32_t* doc_starts, int32_t n_doc_starts, void* O, void* stream) {
  ipttt_status rc = check_params(p);
  if (rc != IPTTT_OK) return rc;
  if (layout_of(*p).total > IPTTT_NOALLOC_SCRATCH_BYTES) return IPTTT_ERR_SHAPE;
  void* ws = nullptr;
  if ((rc = noalloc_scratch(&ws)) != IPTTT_OK) return rc;
  return ipttt_forward(p, H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget, doc_starts, n_doc_starts, O, ws,
                       IPTTT_NOALLOC_SCRATCH_BYTES, stream);
}

void ipttt_profile_enable(int on) { g_profile_on.store(on ? 1 : 0); }

int ipttt_profile_read(double* ms, uint64_t* launches, int n_phases) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  for (auto& pd : g_prof.pending) {
    float e = 0.0f;
    if (cudaEventSynchronize(pd.b) == cudaSuccess && cudaEventElapsedTime(&e, pd.a, pd.b) == cudaSuccess) {
      g_prof.ms[pd.phase] += e;
      g_prof.launches[pd.phase] += pd.launches;
    }
    g_prof.pool.push_back(pd.a);
    g_prof.pool.push_back(pd.b);
  }
  g_prof.pending.clear();
  const int n = n_phases < kPhases ? n_phases : kPhases;
  for (int i = 0; i < n; ++i) {
    if (ms) ms[i] = g_prof.ms[i];
    if (launches) launches[i] = g_prof.launches[i];
    g_prof.ms[i] = 0.0;
    g_prof.launches[i] = 0;
  }
  return n < 0 ? 0 : n;
}

uint64_t ipttt_kernel_launches(void) { return g_launches.load(); }

ipttt_status ipttt_selftest_wait_timeout(uint32_t limit_ns, void* stream) {
  DeviceInfo* di = nullptr;
  ipttt_status rc = device_info(&di);
  if (rc != IPTTT_OK) return rc;
  const uint64_t lim = limit_ns ? limit_ns : 2000000000ull;
  rc = cuda_status(tck::launch_wait_timeout(di->status, lim, static_cast<cudaStream_t>(stream)));
  if (rc == IPTTT_OK) counted(1);
  return rc;
}

}  // extern "C"
