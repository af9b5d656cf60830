// Router: logits = x W_r (+ bias), softmax, top-K with ties to the lower expert id.
//
// "Two upstream innovations of MoE: Routing-Free and OmniMoE" (chatdocs.ruinique.com),
// section 1.1: x -> Router(x) -> Softmax -> TopK. "How AI chips support MoE", chapter 4,
// section 4.2: the gate is a small dense linear map every token passes through; 4.3: the
// top-K is a partial sort per token.
//
// From x: one CTA owns TM tokens. Phase 1 is a register-tiled fp32 FMA GEMM (x tile and W_r
// tile staged through shared memory, fp32 accumulation) that leaves the TM x E logits in
// shared memory. Given logits skip phase 1 and shared memory: a warp loads its tokens' logits
// straight into registers, all of them before the first is ranked, over enough CTAs to
// spread a small batch across the SMs. Phase 2 gives one warp per token: each
// lane holds E/32 logits in registers and the top-K under the total order (value descending,
// id ascending) comes from K rounds of a warp arg-max or, for E <= 64 and K <= 8, from the
// bitonic merges of the lanes' sorted lists (moe_shape.route_topk). Selection compares fp32
// logits, so +0 and -0 tie. Weights: exp(l - l_max) over the selected (renormalised) or over
// all E.
#include <math.h>

#include "common.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kDK = 64;

template <typename Tin, int CT, int CPT, int RPT, int FORM>
__global__ void __launch_bounds__(kThreads) route_kernel(
    const Tin* __restrict__ x, const Tin* __restrict__ w_r, const float* __restrict__ bias,
    float* __restrict__ logits_out, int32_t* __restrict__ topk_ids, float* __restrict__ topk_w,
    int T, int d, int E, int K, int renorm) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  constexpr int RT = kThreads / CT;
  constexpr int TM = RT * RPT;
  constexpr int EP = CT * CPT;
  constexpr int LDL = EP + 1;
  constexpr int VPL = (EP + 31) / 32;
  extern __shared__ float smem[];
  float* lg = smem;  // [TM][LDL]
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * TM;

  {
    constexpr int VEC = Vec16<Tin>::N;
    float* xs = lg + TM * LDL;          // [TM][kDK + 1]
    float* ws = xs + TM * (kDK + 1);    // [kDK][EP]
    const int tc = tid % CT, tr = tid / CT;
    float acc[RPT][CPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int j = 0; j < CPT; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < d; k0 += kDK) {
      // x tile: TM rows x kDK columns, 16-byte vector loads (d is a multiple of kDK)
      for (int i = tid; i < TM * (kDK / VEC); i += kThreads) {
        const int r = i / (kDK / VEC), c = (i % (kDK / VEC)) * VEC;
        const int t = t0 + r;
        float f[VEC];
        if (t < T) {
          const uint4 u = *reinterpret_cast<const uint4*>(x + (size_t)t * d + k0 + c);
          unpack16(u, f, Tin());
        } else {
#pragma unroll
          for (int v = 0; v < VEC; ++v) f[v] = 0.f;
        }
#pragma unroll
        for (int v = 0; v < VEC; ++v) xs[r * (kDK + 1) + c + v] = f[v];
      }
      // W_r tile: kDK rows x EP columns (zero past E)
      for (int i = tid; i < kDK * EP; i += kThreads) {
        const int r = i / EP, c = i % EP;
        ws[i] = (c < E) ? to_f32(w_r[(size_t)(k0 + r) * E + c]) : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int k = 0; k < kDK; ++k) {
        float a[RPT], b[CPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i) a[i] = xs[(tr + i * RT) * (kDK + 1) + k];
#pragma unroll
        for (int j = 0; j < CPT; ++j) b[j] = ws[k * EP + tc + j * CT];
#pragma unroll
        for (int i = 0; i < RPT; ++i)
#pragma unroll
          for (int j = 0; j < CPT; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i)
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const int e = tc + j * CT;
        const float bb = (bias != nullptr && e < E) ? bias[e] : 0.f;
        lg[(tr + i * RT) * LDL + e] = acc[i][j] + bb;
      }
  }
  __syncthreads();

  if (logits_out != nullptr) {
    for (int i = tid; i < TM * E; i += kThreads) {
      const int r = i / E, c = i % E;
      const int t = t0 + r;
      if (t < T) logits_out[(size_t)t * E + c] = lg[r * LDL + c];
    }
  }

  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < TM; r += kThreads / 32) {
    const int t = t0 + r;
    if (t >= T) break;
    float v[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane + 32 * j;
      v[j] = (e < E) ? lg[r * LDL + e] : -INFINITY;
    }
    int sele;
    float selw;
    warp_route_token<VPL, FORM>(v, E, K, renorm, sele, selw);
    if (lane < K) {
      topk_ids[(size_t)t * K + lane] = sele;
      topk_w[(size_t)t * K + lane] = selw;
    }
  }
}

// Given logits: warp w of CTA b ranks tokens (8 b + w) TPW ... + TPW - 1.
template <int VPL, int TPW, int FORM>
__global__ void __launch_bounds__(kThreads) route_given_kernel(
    const float* __restrict__ logits_in, float* __restrict__ logits_out,
    int32_t* __restrict__ topk_ids, float* __restrict__ topk_w, int T, int E, int K, int renorm) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tw0 = ((long long)blockIdx.x * (kThreads / 32) + warp) * TPW;
  float v[TPW][VPL];
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    const long long t = tw0 + i;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane + 32 * j;
      v[i][j] = (t < T && e < E) ? logits_in[t * E + e] : -INFINITY;
    }
  }
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    const long long t = tw0 + i;
    if (t >= T) break;  // warp-uniform
    if (logits_out != nullptr && logits_out != logits_in) {
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int e = lane + 32 * j;
        if (e < E) logits_out[t * E + e] = v[i][j];
      }
    }
    int sele;
    float selw;
    warp_route_token<VPL, FORM>(v[i], E, K, renorm, sele, selw);
    if (lane < K) {
      topk_ids[t * K + lane] = sele;
      topk_w[t * K + lane] = selw;
    }
  }
}

template <int VPL>
moe_status launch_route_given_v(const moe_shape& s, const float* logits_in, float* logits_out,
                                int32_t* ids, float* w, cudaStream_t st) {
  const bool bitonic = VPL <= 2 && route_topk_form(s.route_topk, s.E, s.K) == TOPK_BITONIC;
  // one token a warp while that leaves CTAs for fewer than four waves of the SMs, else four
  const bool four = (long long)s.T >= 4LL * 8 * 4 * sm_count();
  const int tpw = four ? 4 : 1;
  const long long grid = ((long long)s.T + 8LL * tpw - 1) / (8LL * tpw);
  auto launch = [&](auto kern) {
    launch_begin(K_ROUTE, st);
    launch_kernel(kern, dim3((unsigned)grid), dim3(kThreads), 0, st, 1, logits_in, logits_out,
                  ids, w, s.T, s.E, s.K, s.renormalize);
    return launch_end(K_ROUTE, st);
  };
  if (bitonic)
    return four ? launch(route_given_kernel<VPL, 4, TOPK_BITONIC>)
                : launch(route_given_kernel<VPL, 1, TOPK_BITONIC>);
  return four ? launch(route_given_kernel<VPL, 4, TOPK_ROUNDS>)
              : launch(route_given_kernel<VPL, 1, TOPK_ROUNDS>);
}

moe_status launch_route_given(const moe_shape& s, const float* logits_in, float* logits_out,
                              int32_t* ids, float* w, cudaStream_t st) {
  if (s.E <= 32) return launch_route_given_v<1>(s, logits_in, logits_out, ids, w, st);
  if (s.E <= 64) return launch_route_given_v<2>(s, logits_in, logits_out, ids, w, st);
  if (s.E <= 128) return launch_route_given_v<4>(s, logits_in, logits_out, ids, w, st);
  return launch_route_given_v<8>(s, logits_in, logits_out, ids, w, st);
}

template <typename Tin, int CT, int CPT, int RPT>
moe_status launch_route_t(const moe_shape& s, const void* x, const void* w_r, const float* bias,
                          float* logits_out, int32_t* ids, float* w, cudaStream_t st) {
  constexpr int RT = kThreads / CT;
  constexpr int TM = RT * RPT;
  constexpr int EP = CT * CPT;
  const size_t smem =
      ((size_t)TM * (EP + 1) + (size_t)TM * (kDK + 1) + (size_t)kDK * EP) * sizeof(float);
  const bool bitonic = route_topk_form(s.route_topk, s.E, s.K) == TOPK_BITONIC;
  auto kern = bitonic ? route_kernel<Tin, CT, CPT, RPT, TOPK_BITONIC>
                      : route_kernel<Tin, CT, CPT, RPT, TOPK_ROUNDS>;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  const int grid = (s.T + TM - 1) / TM;
  if (grid == 0) return MOE_OK;
  launch_begin(K_ROUTE, st);
  launch_kernel(kern, dim3((unsigned)grid), dim3(kThreads), smem, st, 1, (const Tin*)x,
                (const Tin*)w_r, bias, logits_out, ids, w, s.T, s.d, s.E, s.K, s.renormalize);
  return launch_end(K_ROUTE, st);
}

template <typename Tin>
moe_status launch_route_dt(const moe_shape& s, const void* x, const void* w_r, const float* bias,
                           float* lo, int32_t* ids, float* w, cudaStream_t st) {
  if (s.E <= 8) return launch_route_t<Tin, 8, 1, 2>(s, x, w_r, bias, lo, ids, w, st);
  if (s.E <= 16) return launch_route_t<Tin, 16, 1, 4>(s, x, w_r, bias, lo, ids, w, st);
  if (s.E <= 32) return launch_route_t<Tin, 32, 1, 8>(s, x, w_r, bias, lo, ids, w, st);
  if (s.E <= 64) return launch_route_t<Tin, 32, 2, 8>(s, x, w_r, bias, lo, ids, w, st);
  if (s.E <= 128) return launch_route_t<Tin, 32, 4, 4>(s, x, w_r, bias, lo, ids, w, st);
  return launch_route_t<Tin, 32, 8, 2>(s, x, w_r, bias, lo, ids, w, st);
}

}  // namespace

moe_status launch_route(const moe_shape& s, const void* x, const void* w_r, const float* bias,
                        const float* logits_in, float* logits_out, int32_t* ids, float* w,
                        cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  if (logits_in != nullptr) return launch_route_given(s, logits_in, logits_out, ids, w, st);
  if (s.dtype == MOE_BF16) return launch_route_dt<bf16>(s, x, w_r, bias, logits_out, ids, w, st);
  return launch_route_dt<float>(s, x, w_r, bias, logits_out, ids, w, st);
}

}  // namespace moe
