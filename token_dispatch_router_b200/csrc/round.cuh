// Tile-aware token rounding up or to the nearest tile: limits shared by the host checks and
// the kernels (permute.cu).
#pragma once

namespace moe {

// The selection kernel keeps a bitmap of the tokens routed to its expert in shared memory
// (16 KB at this bound).
constexpr int kRoundUpMaxTokens = 131072;

}  // namespace moe
