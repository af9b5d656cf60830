// Kernel ids of the library's opt-in event profiler: host-side bookkeeping only (no device
// code depends on them).
#pragma once

namespace moe {

// Kernel ids of the opt-in profiler (order = moe_kernel_name).
enum KernelId {
  K_ROUTE = 0,
  K_HIST,
  K_SCAN,
  K_SCATTER,
  K_GATHER,
  K_GATEUP_TC,
  K_DOWN_TC,
  K_GATEUP_SIMT,
  K_DOWN_SIMT,
  K_COMBINE,
  K_SELFTEST,
  K_ROUTE_TC,
  K_PERMUTE_SMALL,
  K_GATEUP_TC2,
  K_DOWN_TC2,
  K_PERMUTE_CLUSTER,
  K_TILE_ROUND,
  K_BWD_ACT,
  K_BWD_DW,
  K_BWD_DX,
  K_ROUTER_DLOGITS,
  K_ROUTER_DWR,
  K_ROUTER_DX,
  K_OMNI_LOGITS,
  K_OMNI_TOPK,
  K_OMNI_COUNT,
  K_OMNI_SCAN,
  K_OMNI_SCATTER,
  K_OMNI_SORT,
  K_OMNI_ACT,
  K_OMNI_OUT,
  K_COUNT
};

}  // namespace moe
