// Weighted combine back to token order.
//
// SonicMoE explainer (gitcode.csdn.net), section 3 item 6: scatter/combine back to the
// token-major layout; section 6.1: the aggregation kernel fuses the scatter and the sum.
//   out[t] = sum_{k, assign_to_perm[t*K+k] >= 0} topk_w[t,k] * y_perm[assign_to_perm[t*K+k]]
// fp32 accumulation in k order (deterministic); dropped slots add nothing. With no weights
// (topk_w NULL, the backward's scatter-add of the input gradient) every slot counts once.
// After token rounding up, a token's added assignments follow its K slots, in expert order.
//
// HBM-bound. One warp owns a 2 KB segment (128 16-byte vectors) of one token's output row:
// the token's K slots and weights are loaded once per lane (same addresses across the warp),
// then for each pair of slots every lane issues eight independent 128-bit loads (4 vectors
// x 2 rows; every warp-wide load covers 512 contiguous bytes), accumulates in fp32 in slot
// order, and writes its four vectors. The rows are read with an L2 evict-first policy: each
// is read exactly once.
#include "common.cuh"

namespace moe {

namespace {

// Added assignments of token rounding up (all NULL otherwise): token t's are idx[ptr[t] ..
// ptr[t+1]) into the added list, in expert order, each with its slot a2p[j] and weight w[j].
struct AddedSlots {
  const int32_t* ptr;
  const int32_t* idx;
  const float* w;
  const int32_t* a2p;
};

template <typename Tv>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ a2p,
                                                      const float* __restrict__ topk_w, int T,
                                                      int K, int vec_per_row, long long n_rows,
                                                      uint4* __restrict__ out, unsigned* status,
                                                      const AddedSlots adds) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  constexpr int V = Vec16<Tv>::N;
  const int segs = (vec_per_row + 127) / 128;
  const long long units = (long long)T * segs;
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  const uint64_t once = l2_policy_evict_first();  // each row is read exactly once
  for (long long u = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units;
       u += warps) {
    const long long t = u / segs;
    const int v0 = (int)(u - t * segs) * 128 + lane;
    float acc[4][V];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < V; ++q) acc[j][q] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 2) {
      long long p[2];
      float w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        p[h] = -1;
        w[h] = 0.f;
        if (k0 + h < K) {
          p[h] = a2p[t * K + k0 + h];
          if (p[h] >= n_rows) {
            if (lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
            p[h] = -1;
          }
          if (p[h] >= 0) w[h] = topk_w != nullptr ? topk_w[t * K + k0 + h] : 1.f;
        }
      }
      uint4 r[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (p[h] >= 0 && v0 + 32 * j < vec_per_row)
            r[h][j] = ld_global_hint(y_perm + p[h] * vec_per_row + v0 + 32 * j, once);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (p[h] < 0) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (v0 + 32 * j >= vec_per_row) continue;
          float f[V];
          unpack16(r[h][j], f, Tv());
#pragma unroll
          for (int q = 0; q < V; ++q) acc[j][q] = fmaf(w[h], f[q], acc[j][q]);
        }
      }
    }
    if (adds.ptr != nullptr) {  // the token's added assignments, in expert order
      for (int i = adds.ptr[t]; i < adds.ptr[t + 1]; ++i) {
        const int j = adds.idx[i];
        long long p = adds.a2p[j];
        if (p >= n_rows) {
          if (lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
          p = -1;
        }
        if (p < 0) continue;
        const float w = adds.w[j];
        uint4 r[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (v0 + 32 * q < vec_per_row) r[q] = ld_global_hint(y_perm + p * vec_per_row + v0 + 32 * q, once);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (v0 + 32 * q >= vec_per_row) continue;
          float f[V];
          unpack16(r[q], f, Tv());
#pragma unroll
          for (int c = 0; c < V; ++c) acc[q][c] = fmaf(w, f[c], acc[q][c]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (v0 + 32 * j < vec_per_row) out[t * vec_per_row + v0 + 32 * j] = pack16(acc[j], Tv());
  }
}

}  // namespace

moe_status launch_combine_added(const moe_shape& s, const void* y_perm, const int32_t* a2p,
                                const float* topk_w, void* out, const int32_t* add_ptr,
                                const int32_t* add_idx, const float* add_w, long long n_rows,
                                cudaStream_t st) {
  const int elem = (s.dtype == MOE_BF16) ? 2 : 4;
  const int vec_per_row = s.d * elem / 16;
  const long long units = (long long)s.T * ((vec_per_row + 127) / 128);  // one warp each
  if (units == 0) return MOE_OK;
  long long blocks = (units + 7) / 8;
  const long long cap_blocks = (long long)sm_count() * 8;
  if (blocks > cap_blocks) blocks = cap_blocks;
  const AddedSlots adds{add_ptr, add_idx, add_w,
                        add_ptr != nullptr ? a2p + (size_t)s.T * s.K : nullptr};
  launch_begin(K_COMBINE, st);
  if (s.dtype == MOE_BF16)
    launch_kernel(combine_kernel<bf16>, dim3((unsigned)blocks), dim3(256), 0, st, 1,
                  (const uint4*)y_perm, a2p, topk_w, s.T, s.K, vec_per_row, n_rows, (uint4*)out,
                  device_status_ptr(), adds);
  else
    launch_kernel(combine_kernel<float>, dim3((unsigned)blocks), dim3(256), 0, st, 1,
                  (const uint4*)y_perm, a2p, topk_w, s.T, s.K, vec_per_row, n_rows, (uint4*)out,
                  device_status_ptr(), adds);
  return launch_end(K_COMBINE, st);
}

moe_status launch_combine(const moe_shape& s, const void* y_perm, const int32_t* a2p,
                          const float* topk_w, void* out, cudaStream_t st) {
  return launch_combine_added(s, y_perm, a2p, topk_w, out, nullptr, nullptr, nullptr,
                              (long long)s.T * s.K, st);
}

}  // namespace moe
