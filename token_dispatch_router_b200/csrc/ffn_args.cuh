// Arguments shared by the single-CTA and CTA-pair grouped-GEMM kernels, and the host
// helper that encodes their TMA tensor maps.
#pragma once

#include "common.cuh"

namespace moe {

struct GemmArgs {
  const int32_t* offsets;  // [E + 1] expert-major row offsets
  const int32_t* p2a;      // gate/up: slot -> flat assignment (token = a / K)
  const uint8_t* x;        // gate/up: token rows gathered by cp.async
  long long x_row_bytes;
  bf16* out;
  int ld_out;    // elements per output row
  int n_out;     // valid output columns
  int out_tile;  // output columns per tile (128 gate/up, 256 down)
  int n_tiles;
  int kblocks;   // contraction / 64
  int kb_split;  // backward dX: k-blocks below it read the first B map, the rest the second
  int E, K, T;
  unsigned* status;
  unsigned long long limit_ns;
  bf16* h_out;  // gate/up, single CTA: if not NULL, also the pre-activations (g | u) per row
};

// bf16 tensor of `rank` dims (innermost first), 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box);

}  // namespace moe
