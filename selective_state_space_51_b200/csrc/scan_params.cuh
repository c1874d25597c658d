// Launch parameters shared by the scan kernels (plain pointers and sizes).
#pragma once

#include <stdint.h>

namespace ssm {

struct ScanParams {
  const void *x;             // [b, L, E] activation dtype (the convolution's
                             // input v when conv_weight is set)
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
  int write_zoh;             // exact zero-order-hold write (see ssm_scan.h)
  // Causal depthwise convolution in front of the scan: x = SiLU(conv_bias +
  // sum_k conv_weight[e, k] v[t - K + 1 + k]), zeros before t = 0.
  const float *conv_weight;  // [E, K] or nullptr (x is used as it is)
  const float *conv_bias;    // [E] or nullptr
  int conv_width;            // K, 1..kScanConvMaxWidth
  // Training forward (unsplit, one time block): the state before every
  // kCkptSteps-th step goes to ckpt [b, ceil(L / kCkptSteps), E, N]; y may
  // then be nullptr (not written).
  float *ckpt;
  // Split sequences (chunked variant): each sequence is cut into `segments`
  // pieces of seg_len steps (a multiple of the window), scanned concurrently
  // from a zero state and joined by a decoupled look-back over per-piece
  // affine aggregates in the workspace below.
  int segments;              // pieces per sequence (1 = no split)
  int64_t seg_len;           // steps per piece
  unsigned *flags;           // [b, segments, tiles] publication words
  float *agg_state;          // [b, segments, E, N] end state from zero
  float *agg_decay;          // [b, segments, E, N] product of retentions
  float *incl_state;         // [b, segments, E, N] true end state
  unsigned *ticket;          // launch-order counter, zero before the launch
  int *status;               // device status word (kStatus*)
  unsigned epoch;            // tag of this call in the publication words
  unsigned spin_limit;       // bounded wait: polls before giving up
  unsigned debug;            // kDebug* bits (tests only)
};

// Steps between the forward checkpoints the backward pass restarts from.
constexpr int kCkptSteps = 8;

// Widest causal convolution the fused scan takes.
constexpr int kScanConvMaxWidth = 4;

// Device status codes written to ScanParams::status.
enum { kStatusOk = 0, kStatusTimeout = 1 };

// Publication states (low 2 bits of a flag word; the rest is the epoch).
enum { kFlagNone = 0, kFlagAggregate = 1, kFlagInclusive = 2 };

// Test hooks: the first piece of every sequence never publishes, so its
// successor's bounded wait must run out and report kStatusTimeout; the
// decode step uses its per-thread-load kernel instead of the bulk-copy one.
enum {
  kDebugNoPublish = 1u << 0,
  kDebugStepPerThread = 1u << 1,
  // the specialised scan runs on persistent blocks wherever it can, in
  // chunks of kDynTestChunk steps (tests of the chunk hand-over on small
  // shapes); kDebugNoDyn: never
  kDebugForceDyn = 1u << 2,
  kDebugNoDyn = 1u << 3
};
// Steps per chunk of the persistent-block scan, and in its forced test mode.
constexpr int64_t kDynChunk = 512;
constexpr int64_t kDynTestChunk = 64;

}  // namespace ssm
