// Launch parameters shared by the scan kernels (plain pointers and sizes).
#pragma once

#include <stdint.h>

namespace ssm {

struct ScanParams {
  const void *x;             // [b, L, E] activation dtype
  const void *delta;         // [b, L, E]
  const float *A_log;        // [E, N]
  const void *B;             // [b, L, N]
  const void *C;             // [b, L, N]
  const float *D;            // [E] or nullptr
  const void *z;             // [b, L, E] or nullptr
  const float *delta_bias;   // [E] or nullptr
  const float *h0;           // [b, E, N] or nullptr
  void *y;                   // [b, L, E]
  float *h_last;             // [b, E, N] or nullptr
  int64_t batch, seqlen, dim;
  int dstate;
  int softplus;              // apply softplus to delta + bias
  // split-sequence workspace (chunked variant with segments > 1)
  int segments;              // pieces per sequence (1 = no split)
  int64_t seg_len;           // steps per piece (multiple of the window)
  float *seg_state;          // [b, segments, E, N] end state from a zero start
  float *seg_decay;          // [b, segments, E, N] product of retentions
  unsigned *seg_flag;        // [b, segments, E / tile] publication flags
  unsigned *ticket;          // [1] launch-order ticket counter
  int *status;               // [1] device status word (0 = ok)
  unsigned epoch;            // value written to flags by this call
};

// Device status codes written to ScanParams::status.
enum { kStatusOk = 0, kStatusTimeout = 1 };

}  // namespace ssm
