// Register top-K helpers shared by the routing kernels: the (value, id) order of the
// selection, a sorted top-KM list per thread with insertion, and the merge of two threads'
// lists over a warp shuffle (a bitonic merge network).
//
// "How AI chips support MoE", chapter 4, section 4.3: top-K is a partial sort per token, and
// for a small number of experts a bitonic network is the natural fixed-structure form.
#pragma once

#include <math.h>

#include "common.cuh"

namespace moe {

// (value, id) order of the selection: a ranks above b when its value is larger, or equal
// (+0 == -0) with a lower id; an empty slot (id < 0) ranks below everything.
__device__ __forceinline__ bool ranks_above(float av, int ae, float bv, int be) {
  if (ae < 0) return false;
  if (be < 0) return true;
  return av > bv || (av == bv && ae < be);
}

// Top-KM list (KM = 2, 4 or 8 >= K), best first, empty slots (id -1) hold -inf. This
// thread's ids arrive in ascending order, so a value equal to a listed one goes below it
// (ties to the lower id, +0 == -0): only a strictly larger value moves an entry down. Slot j
// takes the entry above it when the new value beats both, the new value when it beats slot j
// only, and keeps its own otherwise. Compile-time indices only; the common case, a value
// that does not enter, costs one compare and a branch.
template <int KM>
__device__ __forceinline__ void top_insert(float (&bv)[KM], int (&be)[KM], float v, int e) {
  if (!(v > bv[KM - 1]) && be[KM - 1] >= 0) return;  // does not enter
  bool gt[KM];  // the new value ranks above the entry in slot j
#pragma unroll
  for (int j = 0; j < KM; ++j) gt[j] = be[j] < 0 || v > bv[j];
#pragma unroll
  for (int j = KM - 1; j >= 1; --j) {
    be[j] = gt[j] ? (gt[j - 1] ? be[j - 1] : e) : be[j];
    bv[j] = gt[j] ? (gt[j - 1] ? bv[j - 1] : v) : bv[j];
  }
  if (gt[0]) {
    be[0] = e;
    bv[0] = v;
  }
}

// Merge this thread's sorted list with that of the lane `mask` away (same token group):
// c[i] = better of a[i] and b[KM-1-i] holds the KM best of both lists as a bitonic
// sequence, which log2(KM) half-cleaner stages sort. Both lanes end with the same list.
template <int KM>
__device__ __forceinline__ void top_merge(float (&bv)[KM], int (&be)[KM], int mask) {
  float ov[KM];
  int oe[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    ov[j] = __shfl_xor_sync(0xffffffffu, bv[j], mask);
    oe[j] = __shfl_xor_sync(0xffffffffu, be[j], mask);
  }
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (!ranks_above(bv[j], be[j], ov[KM - 1 - j], oe[KM - 1 - j])) {
      bv[j] = ov[KM - 1 - j];
      be[j] = oe[KM - 1 - j];
    }
  }
#pragma unroll
  for (int h = KM / 2; h >= 1; h /= 2) {
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if ((j & h) == 0) {
        if (ranks_above(bv[j + h], be[j + h], bv[j], be[j])) {
          const float tv = bv[j];
          const int te = be[j];
          bv[j] = bv[j + h];
          be[j] = be[j + h];
          bv[j + h] = tv;
          be[j + h] = te;
        }
      }
    }
  }
}

// Top-KM of one token's E <= 64 logits held by a warp, lane l holding experts l and l + 32
// (v1 and e1 ignored when l + 32 >= E): the two entries of a lane form a sorted list, and five
// merges over shuffles (lane masks 1, 2, 4, 8, 16, each a bitonic merge network) leave every
// lane with the token's top-KM list, best first (value descending, ties to the lower id).
// log2(32) dependent shuffle steps instead of the K x log2(32) of K rounds of a warp arg-max.
template <int KM>
__device__ __forceinline__ void warp_topk_bitonic(float v0, float v1, int E, float (&bv)[KM],
                                                  int (&be)[KM]) {
  const int e0 = (int)(threadIdx.x & 31), e1 = e0 + 32;
#pragma unroll
  for (int k = 0; k < KM; ++k) {
    bv[k] = -INFINITY;
    be[k] = -1;
  }
  if (e0 < E) {
    bv[0] = v0;
    be[0] = e0;
  }
  if (e1 < E) {  // e1 > e0: it goes first only with a strictly larger value
    if (v1 > bv[0]) {
      bv[1] = bv[0];
      be[1] = be[0];
      bv[0] = v1;
      be[0] = e1;
    } else {
      bv[1] = v1;
      be[1] = e1;
    }
  }
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) top_merge<KM>(bv, be, h);
}

// Top-K forms of the warp-per-token routers (moe_shape.route_topk): K rounds of a warp
// arg-max, or the bitonic merges above (E <= 64, K <= 8).
enum RouteTopkForm { TOPK_ROUNDS = 1, TOPK_BITONIC = 2 };

// The bitonic form where it applies and was asked for; automatic (0) = K rounds of a warp
// arg-max, measured faster on B200 (the five merges of eight-entry lists issue about four
// times the instructions of K <= 8 arg-max rounds).
__host__ __device__ __forceinline__ int route_topk_form(int requested, int E, int K) {
  const bool fits = E <= 64 && K <= 8;
  return requested == TOPK_BITONIC && fits ? TOPK_BITONIC : TOPK_ROUNDS;
}

// The top-KM of a warp's token by the bitonic merges, for lane `lane`: the list's best value
// (every lane) and slot `lane`'s entry (lanes below KM).
template <int KM>
__device__ __forceinline__ void bitonic_select(float v0, float v1, int E, float& vmax,
                                               float& selv, int& sele) {
  const int lane = threadIdx.x & 31;
  float bv[KM];
  int be[KM];
  warp_topk_bitonic<KM>(v0, v1, E, bv, be);
  vmax = bv[0];
#pragma unroll
  for (int k = 0; k < KM; ++k)
    if (lane == k) {
      selv = bv[k];
      sele = be[k];
    }
}

// One token routed by a warp: lane l holds v[j], the logit of expert l + 32 j (-inf past E).
// Selection under (value descending, id ascending; +0 == -0) by K rounds of a warp arg-max
// (FORM = TOPK_ROUNDS) or by the bitonic merges (FORM = TOPK_BITONIC, VPL <= 2, K <= 8); lane
// k < K receives slot k's expert id and weight: exp(l_k - l_max) over the sum for the
// selected experts (renorm) or over all E (plain softmax).
template <int VPL, int FORM>
__device__ __forceinline__ void warp_route_token(const float (&v)[VPL], int E, int K, int renorm,
                                                 int& sel_e, float& sel_w) {
  const int lane = threadIdx.x & 31;
  float vmax = 0.f, selv = 0.f;
  int sele = 0;
  if constexpr (FORM == TOPK_BITONIC && VPL <= 2) {
    const float v1 = VPL > 1 ? v[VPL - 1] : -INFINITY;
    if (K <= 2) bitonic_select<2>(v[0], v1, E, vmax, selv, sele);
    else if (K <= 4) bitonic_select<4>(v[0], v1, E, vmax, selv, sele);
    else bitonic_select<8>(v[0], v1, E, vmax, selv, sele);
  } else {
    bool taken[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) taken[j] = (lane + 32 * j >= E);
    for (int k = 0; k < K; ++k) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int e = lane + 32 * j;
        if (!taken[j] && (v[j] > bv || (v[j] == bv && e < be))) {
          bv = v[j];
          be = e;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
#pragma unroll
      for (int j = 0; j < VPL; ++j)
        if (lane + 32 * j == be) taken[j] = true;
      if (k == 0) vmax = bv;
      if (lane == k) {
        selv = bv;
        sele = be;
      }
    }
  }
  const float ex = (lane < K) ? expf(selv - vmax) : 0.f;
  float den;
  if (renorm) {
    den = ex;
  } else {
    den = 0.f;
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      if (lane + 32 * j < E) den += expf(v[j] - vmax);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  sel_e = sele;
  sel_w = ex / den;
}

}  // namespace moe
