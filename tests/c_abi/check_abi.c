/* Plain C use of libipttt.so through include/ipttt.h: no C++ and no torch types
 * cross the boundary.  Runs without a GPU: size queries and argument checks only
 * (every call below returns before any CUDA call).  Exit status 0 when all hold. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ipttt.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  ipttt_params p;
  memset(&p, 0, sizeof p);
  p.B = 1;
  p.T = 2048;
  p.d = 256;
  p.F = 512;
  p.C = 256;
  p.dtype = IPTTT_BF16;
  p.eta = 1e-3f;
  p.clip_thresh = 1e-5f;
  p.flags = 0;

  expect(strlen(ipttt_version()) >= 5, "version string");
  expect(strcmp(ipttt_strerror(IPTTT_OK), ipttt_strerror(IPTTT_ERR_ARG)) != 0, "distinct error strings");
  expect(ipttt_last_error_detail() != NULL && ipttt_last_error_detail()[0] == 0, "no CUDA error detail yet");

  const size_t ws = ipttt_workspace_size(&p);
  expect(ws > 0 && ws % 256 == 0, "workspace size of a valid shape");
  expect(ipttt_stream_state_size(&p) >= (size_t)p.B * p.d * p.F * 4, "streaming state holds the fp32 state");
  expect(ipttt_forward_host_size(&p, 512, 0) > 0, "host-buffer forward size");
  expect(ipttt_forward_host_size(&p, 500, 0) == 0, "piece length not a multiple of C");
  expect(ipttt_decode_state_size(&p) > 0 && ipttt_decode_host_size(&p) > 0, "decode sizes");

  ipttt_params bad = p;
  bad.C = 96; /* not a multiple of 64: outside the bf16 path */
  expect(ipttt_workspace_size(&bad) == 0, "unsupported shape has no workspace size");

  /* argument errors come back synchronously and launch nothing */
  char host[64];
  void* dev = (void*)(uintptr_t)0x100000; /* never dereferenced: the checks fail first */
  expect(ipttt_forward(&p, NULL, dev, dev, dev, dev, dev, dev, NULL, 0, dev, dev, ws, NULL) == IPTTT_ERR_ARG,
         "forward with a null H");
  expect(ipttt_forward(&bad, dev, dev, dev, dev, dev, dev, dev, NULL, 0, dev, dev, ws, NULL) ==
             IPTTT_ERR_UNSUPPORTED,
         "forward with an unsupported chunk size");
  expect(ipttt_forward_host(&p, NULL, NULL, dev, dev, dev, dev, dev, NULL, 0, NULL, dev, 1u << 30, 512, NULL) ==
             IPTTT_ERR_ARG,
         "host-buffer forward with null host buffers");
  expect(ipttt_decode_reset(&p, NULL, host, NULL) == IPTTT_ERR_ARG, "decode reset without a state");
  expect(ipttt_stream_reset(&bad, dev, NULL) == IPTTT_ERR_UNSUPPORTED, "stream reset, unsupported shape");

  /* context parallelism: the host plan of rank 1 of 2 (shards of 2048 tokens) for a
   * row whose document begins at token 1000 and continues through shard 1 */
  int32_t starts[1] = {1000};
  int32_t local[1] = {-1};
  int32_t n_local = -1;
  int32_t plan[4] = {-1, -1, -1, -1};
  expect(ipttt_cp_workspace_size(&p) > ws, "context-parallel workspace holds every chunk's state");
  expect(ipttt_cp_plan(&p, 2, 1, starts, 1, local, &n_local, plan) == IPTTT_OK, "cp plan");
  expect(n_local == 0 && plan[0] == 1 && plan[1] == 0 && plan[2] == 8 && plan[3] == 1,
         "cp plan: shard continues shard 0's document through all 8 chunks");
  expect(ipttt_cp_plan(&p, 2, 2, starts, 1, local, &n_local, plan) == IPTTT_ERR_ARG, "cp plan, rank out of range");
  expect(ipttt_cp_begin(&p, 2, 0, NULL, 0, NULL, dev, dev, dev, dev, dev, (float*)dev, dev, 1u << 30, NULL) ==
             IPTTT_ERR_ARG,
         "cp begin with a null H");
  expect(ipttt_cp_finish(&p, 2, 0, NULL, 0, dev, dev, (const float*)dev, NULL, NULL, dev, 1u << 30, NULL) ==
             IPTTT_ERR_ARG,
         "cp finish with a null O");

  if (failures == 0) printf("C ABI checks passed\n");
  return failures == 0 ? 0 : 1;
}
