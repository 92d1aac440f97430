// Shared definitions of libipttt: status word, layout of the per-chunk metadata,
// small device helpers.  No kernels here.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ipttt.h"

namespace ipttt {

// The argument checks every entry point runs first (IPTTT_OK or the error code).
ipttt_status validate_params(const ipttt_params* p);

// Kernels report errors they cannot return (bad doc_starts, a bounded wait that
// gave up) by setting a per-device status word, passed to them as a pointer; the
// first error wins.  ipttt_get_status reads and clears it.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Per (row, chunk) metadata, all token indices relative to the row start.
//   first_end : end of the chunk's first document segment
//   last_start: start of the chunk's last document segment
//   cont      : 1 when the chunk's first token continues a document begun earlier
//   has_start : 1 when a document starts anywhere inside the chunk
struct ChunkMeta {
  int32_t first_end;
  int32_t last_start;
  int32_t cont;
  int32_t has_start;
};

struct Shape {
  int B, T, d, F, C, k;   // k = number of chunks per row
};

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// SiLU(x) = x * sigmoid(x): fast exponential for the bf16 path, the accurate one
// for the all-fp32 path.
__device__ __forceinline__ float silu_fast(float x) { return x / (1.0f + __expf(-x)); }
__device__ __forceinline__ float silu_precise(float x) { return x / (1.0f + expf(-x)); }

// Host helpers (implemented in api.cu).
ipttt_status cuda_status(cudaError_t e);
// Tokens per step of the chunk scan: 512 when the bf16 path scans chunks of 64,
// 128 or 256 tokens in groups, else C.  Streaming pieces that are multiples of it give
// one call's result bit for bit.
int scan_unit_tokens(const ipttt_params& p);
// The current device's SM count and the device status word (0 on failure).
int device_sms();
int* device_status();

}  // namespace ipttt
