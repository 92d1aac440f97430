// Host-buffer forward of the layer: H, X0 and O live in host memory, the weights
// on the device.  The sequence goes through the streaming entry points piece by
// piece (a piece is a whole number of chunks, all B rows); the host-to-device copy
// of piece i+1 and the device-to-host copy of piece i-1 run on their own streams
// while piece i computes, two device buffers per tensor alternating.  Streaming
// reproduces one call over the whole sequence exactly (the conv look-ahead and the
// state update both stop at chunk ends, the fp32 state is carried), so the result
// equals ipttt_forward on the same data.
//
// Built on the public entry points only (ipttt_stream_reset / _forward and the
// size queries); nothing of the layer's arithmetic is here.
#include <cuda_runtime.h>

#include <algorithm>
#include <vector>

#include "common.cuh"

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t elem_bytes(const ipttt_params& p) { return p.dtype == IPTTT_BF16 ? 2 : 4; }

// Piece length: the caller's, else about an eighth of the sequence in whole scan
// steps (chunks, or groups of chunks), which keeps the result bit-identical to one
// call over the whole sequence.
int32_t piece_tokens_of(const ipttt_params& p, int32_t piece) {
  if (piece > 0) return piece;
  const int32_t unit = ipttt::scan_unit_tokens(p);
  const int32_t k = (p.T + unit - 1) / unit;
  return std::max<int32_t>(1, k / 8) * unit;
}

struct HostLayout {
  size_t piece;   // bytes of one [B, P, d] piece
  size_t in_h, in_x, out_o, docs, state, ws, ws_bytes, total;
};

bool host_layout(const ipttt_params& p, int32_t P, int32_t n_doc, HostLayout& L) {
  ipttt_params pp = p;
  pp.T = std::min(P, p.T);
  const size_t ws = ipttt_workspace_size(&pp);
  const size_t st = ipttt_stream_state_size(&pp);
  if (ws == 0 || st == 0) return false;
  L.piece = align256((size_t)p.B * pp.T * p.d * elem_bytes(p));
  size_t off = 0;
  L.in_h = off;  off += 2 * L.piece;
  L.in_x = off;  off += 2 * L.piece;
  L.out_o = off; off += 2 * L.piece;
  L.docs = off;  off += align256((size_t)std::max(n_doc, 1) * sizeof(int32_t));
  L.state = off; off += align256(st);
  L.ws = off;    off += align256(ws);
  L.ws_bytes = ws;
  L.total = off;
  return true;
}

// Owns the copy streams and events of one call; releasing them while work is
// still queued is allowed (the driver frees them once it completes).
struct Pipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in_ready[2] = {}, done[2] = {}, out_free[2] = {};
  ~Pipe() {
    if (start) cudaEventDestroy(start);
    for (int i = 0; i < 2; ++i) {
      if (in_ready[i]) cudaEventDestroy(in_ready[i]);
      if (done[i]) cudaEventDestroy(done[i]);
      if (out_free[i]) cudaEventDestroy(out_free[i]);
    }
    if (h2d) cudaStreamDestroy(h2d);
    if (d2h) cudaStreamDestroy(d2h);
  }
  bool create() {
    if (cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&start, cudaEventDisableTiming) != cudaSuccess) return false;
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&in_ready[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&done[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&out_free[i], cudaEventDisableTiming) != cudaSuccess)
        return false;
    return true;
  }
};

}  // namespace

extern "C" {

size_t ipttt_forward_host_size(const ipttt_params* p, int32_t piece_tokens, int32_t n_doc_starts) {
  if (ipttt::validate_params(p) != IPTTT_OK || n_doc_starts < 0) return 0;
  const int32_t P = piece_tokens_of(*p, piece_tokens);
  if (P % p->C != 0) return 0;
  HostLayout L;
  return host_layout(*p, P, n_doc_starts, L) ? L.total : 0;
}

ipttt_status ipttt_forward_host(const ipttt_params* p, const void* H_host, const void* X0_host,
                                const void* Wgate, const void* Wup, const void* Wdown0, const void* conv_w,
                                const void* Wtarget, const int32_t* doc_starts_host, int32_t n_doc_starts,
                                void* O_host, void* device_buffer, size_t device_bytes, int32_t piece_tokens,
                                void* stream) {
  const ipttt_status vrc = ipttt::validate_params(p);
  if (vrc != IPTTT_OK) return vrc;
  if (!H_host || !X0_host || !O_host || !device_buffer || n_doc_starts < 0 ||
      (n_doc_starts > 0 && !doc_starts_host))
    return IPTTT_ERR_ARG;
  const int32_t P = piece_tokens_of(*p, piece_tokens);
  if (P <= 0 || P % p->C != 0) return IPTTT_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(device_buffer) % 256 != 0) return IPTTT_ERR_ALIGN;
  HostLayout L;
  if (!host_layout(*p, P, n_doc_starts, L)) return IPTTT_ERR_SHAPE;
  if (device_bytes < L.total) return IPTTT_ERR_WORKSPACE;

  // Document starts, checked here and split per piece: a start b*T + t inside
  // piece [a, a + len) becomes b*len + (t - a) of that piece.
  const int64_t BT = (int64_t)p->B * p->T;
  const int32_t n_pieces = (p->T + P - 1) / P;
  std::vector<int32_t> local;
  std::vector<int32_t> first(n_pieces + 1, 0);
  local.reserve(n_doc_starts);
  for (int32_t i = 0; i < n_doc_starts; ++i) {
    const int64_t g = doc_starts_host[i];
    if (g < 0 || g >= BT || (i > 0 && g <= doc_starts_host[i - 1])) return IPTTT_ERR_ARG;
  }
  for (int32_t q = 0; q < n_pieces; ++q) {
    const int32_t a = q * P, len = std::min(P, p->T - a);
    first[q] = (int32_t)local.size();
    for (int32_t i = 0; i < n_doc_starts; ++i) {
      const int64_t g = doc_starts_host[i];
      const int32_t b = (int32_t)(g / p->T), t = (int32_t)(g % p->T);
      if (t >= a && t < a + len) local.push_back(b * len + (t - a));
    }
  }
  first[n_pieces] = (int32_t)local.size();

  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  Pipe pipe;
  if (!pipe.create()) return IPTTT_ERR_CUDA;
  uint8_t* base = static_cast<uint8_t*>(device_buffer);
  const size_t es = elem_bytes(*p);
  const size_t row_bytes = (size_t)p->T * p->d * es;  // one host row [T, d]
  void* state = base + L.state;
  int32_t* docs_dev = reinterpret_cast<int32_t*>(base + L.docs);
  const uint8_t* Hh = static_cast<const uint8_t*>(H_host);
  const uint8_t* Xh = static_cast<const uint8_t*>(X0_host);
  uint8_t* Oh = static_cast<uint8_t*>(O_host);

#define IPH_CUDA(x)                                 \
  do {                                              \
    if ((x) != cudaSuccess) return IPTTT_ERR_CUDA;  \
  } while (0)
#define IPH_CALL(x)                      \
  do {                                   \
    const ipttt_status rc_ = (x);        \
    if (rc_ != IPTTT_OK) return rc_;     \
  } while (0)

  // Work already queued on the caller's stream may still use the buffer.
  IPH_CUDA(cudaEventRecord(pipe.start, cs));
  IPH_CUDA(cudaStreamWaitEvent(pipe.h2d, pipe.start, 0));
  IPH_CUDA(cudaStreamWaitEvent(pipe.d2h, pipe.start, 0));
  if (!local.empty())
    IPH_CUDA(cudaMemcpyAsync(docs_dev, local.data(), local.size() * sizeof(int32_t), cudaMemcpyHostToDevice,
                             cs));
  IPH_CALL(ipttt_stream_reset(p, state, stream));

  for (int32_t q = 0; q < n_pieces; ++q) {
    const int s = q & 1;
    const int32_t a = q * P, len = std::min(P, p->T - a);
    const size_t pr = (size_t)len * p->d * es;  // one row of the piece
    uint8_t* dh = base + L.in_h + s * L.piece;
    uint8_t* dx = base + L.in_x + s * L.piece;
    uint8_t* dout = base + L.out_o + s * L.piece;
    // inputs of piece q once piece q-2 has finished reading this buffer
    if (q >= 2) IPH_CUDA(cudaStreamWaitEvent(pipe.h2d, pipe.done[s], 0));
    IPH_CUDA(cudaMemcpy2DAsync(dh, pr, Hh + (size_t)a * p->d * es, row_bytes, pr, p->B, cudaMemcpyHostToDevice,
                               pipe.h2d));
    IPH_CUDA(cudaMemcpy2DAsync(dx, pr, Xh + (size_t)a * p->d * es, row_bytes, pr, p->B, cudaMemcpyHostToDevice,
                               pipe.h2d));
    IPH_CUDA(cudaEventRecord(pipe.in_ready[s], pipe.h2d));
    // compute once the inputs are in and piece q-2's output has left this buffer
    IPH_CUDA(cudaStreamWaitEvent(cs, pipe.in_ready[s], 0));
    if (q >= 2) IPH_CUDA(cudaStreamWaitEvent(cs, pipe.out_free[s], 0));
    ipttt_params pp = *p;
    pp.T = len;
    const int32_t nd = first[q + 1] - first[q];
    IPH_CALL(ipttt_stream_forward(&pp, state, dh, dx, Wgate, Wup, Wdown0, conv_w, Wtarget,
                                  nd > 0 ? docs_dev + first[q] : nullptr, nd, dout, base + L.ws, L.ws_bytes,
                                  stream));
    IPH_CUDA(cudaEventRecord(pipe.done[s], cs));
    // output of piece q back to the host
    IPH_CUDA(cudaStreamWaitEvent(pipe.d2h, pipe.done[s], 0));
    IPH_CUDA(cudaMemcpy2DAsync(Oh + (size_t)a * p->d * es, row_bytes, dout, pr, pr, p->B, cudaMemcpyDeviceToHost,
                               pipe.d2h));
    IPH_CUDA(cudaEventRecord(pipe.out_free[s], pipe.d2h));
  }
  // Later work on the caller's stream sees every copy finished.
  for (int s = 0; s < std::min<int32_t>(2, n_pieces); ++s) IPH_CUDA(cudaStreamWaitEvent(cs, pipe.out_free[s], 0));
#undef IPH_CUDA
#undef IPH_CALL
  return IPTTT_OK;
}

}  // extern "C"
