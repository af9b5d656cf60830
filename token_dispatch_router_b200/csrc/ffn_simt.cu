// fp32 grouped SwiGLU FFN on CUDA cores (FFMA, fp32 accumulation) for MOE_F32 shapes.
//
// SonicMoE explainer (gitcode.csdn.net), section 3 items 3-5: grouped GEMM with a
// different M per expert, SwiGLU, second grouped GEMM; section 6.2: the gather of x by
// routing index happens in the operand load; section 6.3: SwiGLU in the epilogue.
//
// 64x64 output tiles, 256 threads with 4x4 register micro-tiles, 16-deep k slices staged in
// shared memory. The variable-M schedule is built on the device: each CTA reads offsets[],
// derives the per-expert 64-row tile counts and finds its (expert, m-tile) from blockIdx.y;
// CTAs past the last tile exit. No host sync, no atomics.
#include <math.h>

#include "common.cuh"

namespace moe {

namespace {

constexpr int SBM = 64, SBN = 64, SBK = 16, kThreads = 256, kMaxE = 256;

// (expert, first row, valid rows) of global m-tile `mt`; false past the last tile.
__device__ bool find_mtile(const int32_t* offsets, int E, int mt, int* s_off, int* s_cum,
                           int& e, int& row0, int& rows) {
  const int tid = threadIdx.x;
  for (int i = tid; i <= E; i += blockDim.x) s_off[i] = offsets[i];
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int i = 0; i < E; ++i) {
      s_cum[i] = run;
      run += (s_off[i + 1] - s_off[i] + SBM - 1) / SBM;
    }
    s_cum[E] = run;
  }
  __syncthreads();
  if (mt >= s_cum[E]) return false;
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_cum[mid] <= mt) lo = mid;
    else hi = mid - 1;
  }
  e = lo;
  row0 = s_off[e] + (mt - s_cum[e]) * SBM;
  rows = min(SBM, s_off[e + 1] - row0);
  return true;
}

// GATEUP: out[p, :n] = silu(x[tok(p)] Wg[e]) * (x[tok(p)] Wu[e]);  else out[p, :d] = a[p] Wd[e]
template <bool GATEUP>
__global__ void __launch_bounds__(kThreads) ffn_simt_kernel(
    const float* __restrict__ a_src, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ p2a, const float* __restrict__ w0, const float* __restrict__ w1,
    float* __restrict__ out, int E, int K, int T, int kdim, int ncols, unsigned* status) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  __shared__ int s_off[kMaxE + 1], s_cum[kMaxE + 1];
  __shared__ long long s_src[SBM];
  __shared__ float As[SBK][SBM + 4];
  __shared__ float B0[SBK][SBN];
  __shared__ float B1[GATEUP ? SBK : 1][GATEUP ? SBN : 1];
  int e, row0, rows;
  if (!find_mtile(offsets, E, blockIdx.y, s_off, s_cum, e, row0, rows)) return;
  const int n0 = blockIdx.x * SBN;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  if (tid < SBM) {
    long long src = row0;  // row of a_src feeding tile row tid
    if (tid < rows) {
      if (GATEUP) {
        const int a = p2a[row0 + tid];
        const int t = a / K;
        if (a < 0 || t >= T) {
          report(status, MOE_ERR_DEVICE_INDEX);
          src = 0;
        } else {
          src = t;
        }
      } else {
        src = row0 + tid;
      }
    } else {
      src = GATEUP ? 0 : row0;  // padding rows: any valid row, never stored
    }
    s_src[tid] = src;
  }
  __syncthreads();
  const float* w0e = w0 + (size_t)e * kdim * ncols;
  const float* w1e = GATEUP ? w1 + (size_t)e * kdim * ncols : nullptr;
  float acc0[4][4], acc1[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.f;

  for (int k0 = 0; k0 < kdim; k0 += SBK) {
    for (int i = tid; i < SBM * SBK; i += kThreads) {
      const int r = i / SBK, c = i % SBK;
      As[c][r] = a_src[(size_t)s_src[r] * kdim + k0 + c];
    }
    for (int i = tid; i < SBK * SBN; i += kThreads) {
      const int r = i / SBN, c = i % SBN;
      const bool ok = n0 + c < ncols;
      B0[r][c] = ok ? w0e[(size_t)(k0 + r) * ncols + n0 + c] : 0.f;
      if (GATEUP) B1[r][c] = ok ? w1e[(size_t)(k0 + r) * ncols + n0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SBK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b0[j] = B0[kk][tx + 16 * j];
        if (GATEUP) b1[j] = B1[kk][tx + 16 * j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (GATEUP) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty + 16 * i;
    if (r >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx + 16 * j;
      if (c >= ncols) continue;
      float v = acc0[i][j];
      if (GATEUP) {
        const float g = acc0[i][j];
        v = g / (1.f + expf(-g)) * acc1[i][j];
      }
      out[(size_t)(row0 + r) * ncols + c] = v;
    }
  }
}

}  // namespace

moe_status launch_ffn_simt(const moe_shape& s, const void* x, const int32_t* offsets,
                           const int32_t* p2a, const void* w_gate, const void* w_up,
                           const void* w_down, void* a_act, void* y_perm, cudaStream_t st) {
  const long long A = (long long)s.T * s.K;
  if (A == 0) return MOE_OK;
  const long long mtiles = (A + SBM - 1) / SBM + s.E;  // upper bound of sum ceil(kept_e / 64)
  if (mtiles > 65535) return MOE_ERR_UNSUPPORTED;
  unsigned* status = device_status_ptr();
  moe_status r;
  dim3 g1((s.n + SBN - 1) / SBN, (unsigned)mtiles);
  launch_begin(K_GATEUP_SIMT, st);
  launch_kernel(ffn_simt_kernel<true>, g1, dim3(kThreads), 0, st, 1, (const float*)x, offsets, p2a,
                (const float*)w_gate, (const float*)w_up, (float*)a_act, s.E, s.K, s.T, s.d, s.n,
                status);
  if ((r = launch_end(K_GATEUP_SIMT, st)) != MOE_OK) return r;
  dim3 g2((s.d + SBN - 1) / SBN, (unsigned)mtiles);
  launch_begin(K_DOWN_SIMT, st);
  launch_kernel(ffn_simt_kernel<false>, g2, dim3(kThreads), 0, st, 1, (const float*)a_act, offsets,
                p2a, (const float*)w_down, (const float*)nullptr, (float*)y_perm, s.E, s.K, s.T,
                s.n, s.d, status);
  return launch_end(K_DOWN_SIMT, st);
}

}  // namespace moe
