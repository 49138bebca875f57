// tc.h -- parameters of the tensor-core dequant-GEMM kernel (tc.cu).
#pragma once

#include <cuda.h>

#include "pw_internal.h"

namespace pw {

constexpr int kTcTokens = 32;   // decode token tile of one work item (MMA N <= 32)
constexpr int kTcPfTokens = 256;  // prefill token chunk of one work item (MMA N = 256)
// decode modes (token tiles of up to 32 rows)
constexpr int kTcGateUp = 0;    // gate and up blocks of every group -> h = silu(g) * u
constexpr int kTcDown = 1;      // down blocks, B = h -> routing-weighted partials
constexpr int kTcLinear = 2;    // one standalone block -> y
// prefill modes (256-token chunks; gate and up in separate launches)
constexpr int kTcPfGate = 3;    // gate blocks -> g (fp16, gbuf)
constexpr int kTcPfUp = 4;      // up blocks -> h = silu(g) * u (h_perm)
constexpr int kTcPfDown = 5;    // down blocks -> routing-weighted outputs (ysorted)
// decode, both passes in one launch: gate/up items, then down items; a down
// item of group g starts loading h once g's gate/up items are all written
constexpr int kTcFused = 6;

struct TcParams {
  CUtensorMap b_maps[4];         // token-tile source (modes 0, 1): x_sorted or h_perm
                                 // as {64 columns, rows, atoms}; box i holds 8(i+1)
                                 // rows x 2 atoms, 128-byte swizzle
  CUtensorMap pf_map;            // prefill modes: the same source, box 256 rows x 1 atom
  CUtensorMap h_maps[4];         // fused mode: the down items' source (h_perm)
  PageTable pt;                  // planes, bits, active LUT slot per block (modes 0, 1)
  int mode;
  int H, F, S, E, n_groups, n_max;
  int n_split;                   // K ranges of the down pass (1 otherwise)
  const int32_t* offsets;        // [G+1] sorted-position ranges per group
  const int32_t* slot_token;
  const float* slot_w;
  const uint16_t* x;             // bf16 activations [T][lin_cols] (mode 2)
  uint16_t* h_perm;              // fp16 silu(g)*u in the A K order, atom-major
  int h_perm_ld, h_rows;         // [h_perm_ld/64][h_rows][64] (written by mode 0,
                                 // read by mode 1; zero past F)
  float* ysorted;                // [n_split][P][H]
  long long split_stride;        // floats between split partial buffers
  float* y;                      // [T][lin_rows] (mode 2)
  int T;
  int lin_rows, lin_cols, lin_bits, lin_n_max;
  const uint16_t* lin_lut;
  const uint32_t* lin_planes;    // plane pages of the standalone block (mode 2)
  int* gu_done;                   // fused mode: per group, 4 x gate/up items written
                                 // (zero at launch)
  uint16_t* gbuf;                // prefill: gate outputs [rows][gbuf_ld] fp16
  int gbuf_ld;
  int* err;                      // device error word (may be null)
  int cooperative;               // fused mode: launch with the cooperative attribute
  unsigned long long wait_ns;    // limit of one device-side wait (0: 2 s)
  int test_stall_group;          // test switch: this group's down items wait for
                                 // a count that never arrives (-1: off)
};

cudaError_t launch_tc(const TcParams& p, int n_sm, cudaStream_t s);

}  // namespace pw
