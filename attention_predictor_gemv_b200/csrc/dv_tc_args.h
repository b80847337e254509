// Argument blocks and sizes of the tensor-core gathered-row kernels
// (dv_tc.cuh), shared by the kernels and the host code that launches them.
#pragma once

#include <cuda.h>  // CUtensorMap
#include <cuda_bf16.h>
#include <stdint.h>

namespace dv {

constexpr int TC_M = 128;         // tile rows (rowdot) / columns (rowaxpy)
constexpr int TC_N = 16;          // batch rows, zero-padded
constexpr int TC_MIN_B = 5;       // batch rows from which the layer calls use the tensor-core kernels
constexpr int TC_MAX_TILES = 1024;  // tiles of 128 selected neurons (k_max <= 131072)
constexpr int DV_DEV_TIMEOUT_BIT = 8;  // device status bit: a bounded wait ran out

// TMA descriptors of one kernel (128-byte swizzle, bf16): the weight rows
// (boxes of 64 columns x 1 row for gathered rows, 64 x 64 for W^O) and the
// operand's hi and lo rows [16][ld] (boxes of 64 x 16).
struct TcMaps {
  CUtensorMap w, hi, lo;
  CUtensorMap w2;  // a second weight matrix (the dense rowdot's second row block)
};

struct TcQkvArgs {
  const __nv_bfloat16* Wqkv;  // [h][3][dh][d]
  const float* bqkv;          // [h][3][dh] or null
  const __nv_bfloat16* xhi;   // [16][d] normalised input, hi part (rows >= nb zero)
  const __nv_bfloat16* xlo;   // [16][d] lo part
  const int32_t* head_idx;
  const int32_t* head_count;
  int kh_max, h, dh, d, nb, cap, pos;
  float* q;                   // [nb][kh_max][dh]
  __nv_bfloat16* Kc;          // [nb][h][cap][dh]
  __nv_bfloat16* Vc;
  int* status;
  float* red;                 // [tiles][parts][16][128] split-K partial sums (parts <= 8)
  unsigned* tick;             // [tiles] parts finished per tile, zero between calls
  int stages;                 // ring stages (set by the launcher)
};

struct TcMlpArgs {
  const __nv_bfloat16* W1t;  // [N][d]
  const float* b1;           // [N]
  const __nv_bfloat16* W2t;  // [N][d]
  const float* b2;           // [d] or null
  const __nv_bfloat16* xhi;  // [16][d] normalised input, hi part
  const __nv_bfloat16* xlo;  // [16][d] lo part
  const int32_t* idx;
  const int32_t* count;
  int k_max, d, N, nb;
  int KC;                    // slots per batch row of act_c: tiles_max x 128
  int tiles_per_group;       // rowdot tiles per rowaxpy unit
  __nv_bfloat16* act_hi;     // [16][KC] activations compacted per tile, hi part
  __nv_bfloat16* act_lo;     // [16][KC] lo part
  int32_t* rowid_c;          // [KC] the neuron of each compacted slot
  int32_t* tile_cnt;         // [tiles_max] nonzero neurons per tile
  float* out;                // [nb][d], accumulated into
  int* status;
  int act;                   // ACT_RELU or ACT_GELU
  float* red;                // [tiles][parts][16][128] split-K partial sums of W1 (parts <= 8)
  unsigned* tick;            // [tiles] parts finished per tile, zero between calls
  unsigned long long* acc;   // [nb][d] fixed-point partial sums of W2, zero between calls
  int stages;                // ring stages (set by the launcher)
};

struct TcWoArgs {
  const __nv_bfloat16* WOt;  // [h][dh][d]
  const float* bO;           // [d] or null
  const __nv_bfloat16* hhi;  // [16][kh_max dh] attention outputs H, hi part
  const __nv_bfloat16* hlo;  // lo part
  const int32_t* head_idx;
  const int32_t* head_count;
  int kh_max, h, dh, d, nb;
  int heads_per_group;
  float* out;                // [nb][d], accumulated into
  int* status;
  unsigned long long* acc;   // [nb][d] fixed-point partial sums, zero between calls
  int stages;                // ring stages (set by the launcher)
};

// Dense rowdot over consecutive rows of up to two matrices sharing the
// operand (the predictor's GEMMs at batch >= 3): out1[b][i] = W1[i] . X[b]
// (+ bias1[i]) for i < n1 (maps.w), then out2[b][i] = W2[i] . X[b] (+
// bias2[i]) for i < n2 (maps.w2); the first block is padded to p1 =
// ceil(n1 / 64) 64 rows, so a 64-row tile never spans both.
struct TcDenseArgs {
  const float* bias1;  // [n1] or null
  const float* bias2;  // [n2] or null
  int n1, n2, K, nb;
  int kslog;           // log2 of the K splits per 128-row tile
  float* out1;         // [nb][ldo1]
  float* out2;         // [nb][ldo2]
  long long ldo1, ldo2;
  int* status;
  float* red;         // [tiles][2^kslog][16][128] split-K partial sums
  unsigned* tick;     // [tiles] parts finished per tile, zero between calls
  int stages;         // ring stages (set by the launcher)
};

}  // namespace dv
