// Atomic (rank-1) experts behind a Cartesian-product router, run expert-centric.
//
// "Two upstream innovations of MoE: Routing-Free and OmniMoE" (chatdocs.ruinique.com):
// section 2.1 (an expert is a pair of d-vectors, E_i(x) = sigma(x . w_in_i) w_out_i),
// section 2.2 (Cartesian-product router over an N_r x N_c grid: p_r = x W_r, p_c = x W_c,
// score LogSoftmax(p_r)_i + LogSoftmax(p_c)_j), section 2.3 (expert-centric scheduling: the
// (token, expert) tasks sorted by (expert, token), each expert's parameters loaded once for
// all of its tokens), section 3.2 (one scalar per task is the only intermediate; token rows
// are read by id inside the kernel).
//
// Kernels (bf16 tables and activations, fp32 logits, scalars and sums):
//  omni_logits   x [T, d] times W_r [d, N_r] and W_c [d, N_c] on tcgen05 -> logits
//                [T, N_r + N_c] fp32 (row axis first); one 128-token x NT-column tile per CTA.
//  omni_topk     one CTA per token: both axes sorted (value descending, id ascending); the
//                K-th largest pair-sum key is found by a radix select over the "staircase"
//                {(r, c): (r + 1)(c + 1) <= K} of sorted ranks, which holds every pair above
//                it and at least K pairs at or above it; per-row binary searches then give
//                each row's pairs above and at the threshold; pairs at the threshold go to
//                the lowest ids; the K winners are sorted and weighted.
//  omni_count, omni_scan, omni_scatter, omni_segsort, omni_bigsort
//                the task list sorted by (expert, token): counts, offsets, both maps. The
//                scatter claims slots with atomics; each expert's slots are then sorted by
//                assignment id (= by token), so the result is the stable order.
//  omni_act      expert-centric: a warp per expert holds w_in[e] in registers and streams
//                its tokens' rows from L2: h[t K + k] = w_{t,k} silu(x_t . w_in[e]).
//  omni_out      token-centric: y_t = sum_k h[t K + k] w_out[i_{t,k}], rows gathered, k in a
//                fixed order (deterministic; no atomics).
// The pair-sum decision is taken in fp32 on fl(p_r[i] + p_c[j]): the two log-sum-exp terms
// are the same for all pairs of a token, so they do not change the ranking.
#include <math.h>

#include "common.cuh"
#include "ffn_args.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace ptx;

// ------------------------------------------------------------------ logits GEMM
constexpr int LBM = 128, LBK = 64, L_THREADS = 128, L_STAGES = 4;
constexpr int LA_BYTES = LBM * LBK * 2;  // 16 KB: 128 tokens x 64 k
constexpr int LB_CHUNK = LBK * 64 * 2;   // 8 KB: 64 k-rows x 64 columns

struct LogitsArgs {
  float* logits;  // [T, P]
  int T, nr, nc, P, ct_r, kblocks;
  unsigned* status;
  unsigned long long limit_ns;
};

template <int NT>  // columns per tile: 64, 128, 192 or 256
__global__ void __launch_bounds__(L_THREADS) omni_logits_kernel(const __grid_constant__ CUtensorMap tmX,
                                                                const __grid_constant__ CUtensorMap tmR,
                                                                const __grid_constant__ CUtensorMap tmC,
                                                                const LogitsArgs g) {
  constexpr int NCH = NT / 64;
  constexpr int STAGE = LA_BYTES + NCH * LB_CHUNK;
  constexpr uint32_t TCOLS = NT <= 64 ? 64 : (NT <= 128 ? 128 : 256);
  constexpr uint32_t IDESC = idesc_bf16(LBM, NT);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(ring + L_STAGES * STAGE);
  uint64_t* empty = full + L_STAGES;
  uint64_t* accf = empty + L_STAGES;
  uint32_t* tmem_slot = (uint32_t*)(accf + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, j = blockIdx.y;
  const bool col_axis = j >= g.ct_r;
  const int col0 = (col_axis ? j - g.ct_r : j) * NT;
  const CUtensorMap* tmW = col_axis ? &tmC : &tmR;
  const int naxis = col_axis ? g.nc : g.nr;
  const int colbase = (col_axis ? g.nr : 0) + col0;
  const int valid = min(NT, naxis - col0);

  if (tid == 0) {
    for (int s = 0; s < L_STAGES; ++s) {
      mbar_init(saddr(&full[s]), 1);
      mbar_init(saddr(&empty[s]), 1);
    }
    mbar_init(saddr(accf), 1);
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc<1>(saddr(tmem_slot), TCOLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    for (int kb = 0; kb < g.kblocks; ++kb) {
      if (!mbar_wait(saddr(&empty[stage]), phase ^ 1u, nullptr, g.status, g.limit_ns)) break;
      const uint32_t fb = saddr(&full[stage]);
      mbar_expect_tx(fb, STAGE);
      const uint32_t a = saddr(ring + stage * STAGE);
      tma_load_2d(a, &tmX, kb * LBK, tile * LBM, fb);
#pragma unroll
      for (int c = 0; c < NCH; ++c)
        tma_load_2d(a + LA_BYTES + c * LB_CHUNK, tmW, col0 + c * 64, kb * LBK, fb);
      if (++stage == L_STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int kb = 0; kb < g.kblocks; ++kb) {
      if (!mbar_wait(saddr(&full[stage]), phase, nullptr, g.status, g.limit_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a = saddr(ring + stage * STAGE);
#pragma unroll
      for (int kk = 0; kk < LBK / 16; ++kk) {
        const uint64_t ad = desc_sw128(a + kk * 32, 16, 1024);
        const uint64_t bd = desc_sw128(a + LA_BYTES + kk * 2048, LB_CHUNK, 1024);
        tc_mma<1>(tmem, ad, bd, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit<1>(saddr(&empty[stage]));
      if (++stage == L_STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (ok) tc_commit<1>(saddr(accf));
  }
  __syncwarp();
  int w_ok = 0;
  if (lane == 0) w_ok = mbar_wait(saddr(accf), 0, nullptr, g.status, g.limit_ns);
  w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
  tc_fence_after();
  const int r = warp * 32 + lane;
  const int t = tile * LBM + r;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  if (w_ok) {
#pragma unroll 1
    for (int c0 = 0; c0 < NT; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(trow + (uint32_t)c0, v);
      tmem_ld_wait();
      if (t < g.T) {
        float* dst = g.logits + (size_t)t * g.P + colbase + c0;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (c0 + 4 * q < valid)
            *reinterpret_cast<float4*>(dst + 4 * q) =
                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, TCOLS);
  }
}

// ------------------------------------------------------------------ top-K over the grid
constexpr int TK_THREADS = 256;
constexpr int TK_WARPS = TK_THREADS / 32;

// Unsigned key with the order of the float (+0 and -0 equal; NaN assumed absent).
__device__ __forceinline__ uint32_t ord_key(float v) {
  const uint32_t b = __float_as_uint(v == 0.f ? 0.f : v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
// Descending order of composites = value descending, then id ascending.
__device__ __forceinline__ uint64_t composite(uint32_t key, uint32_t id) {
  return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - id);
}

__host__ __device__ inline int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

constexpr int kStairMax = 16384;  // staircase keys kept in shared memory (else recomputed)

// Shared-memory layout of omni_topk (byte offsets), computed on the host and passed in.
// The staircase: row r of the sorted grid keeps columns [0, min(nc, K / (r + 1))), for
// r < min(nr, K); `stair` is its size.
struct TopkSmem {
  int PP, KP;  // padded axis length and padded K (powers of two)
  int stair, stored;  // staircase size; keys kept in shared memory (1) or recomputed (0)
  int o_rk, o_ck, o_sel, o_raw_r, o_raw_c, o_sv_r, o_sv_c, o_sid_r, o_sid_c, o_gt, o_tie,
      o_gpos, o_tpos, o_soff, o_skeys, o_hist, o_misc, total;
};

TopkSmem topk_smem_layout(int nr, int nc, int K) {
  TopkSmem L;
  L.PP = pow2_at_least(max(256, nr > nc ? nr : nc));  // the sorts work on 256 x 2^i keys
  L.KP = pow2_at_least(max(256, K));
  const int R = nr < K ? nr : K;
  long long st = 0;
  for (int r = 0; r < R; ++r) st += (nc < K / (r + 1)) ? nc : K / (r + 1);
  L.stair = (int)st;
  L.stored = st <= kStairMax;
  int o = 0;
  auto take = [&](int bytes) {
    const int at = o;
    o += (bytes + 15) & ~15;
    return at;
  };
  L.o_rk = take(L.PP * 8);
  L.o_ck = take(L.PP * 8);
  L.o_sel = take(L.KP * 8);
  L.o_raw_r = take(nr * 4);
  L.o_raw_c = take(nc * 4);
  L.o_sv_r = take(nr * 4);
  L.o_sv_c = take(nc * 4);
  L.o_sid_r = take(nr * 4);
  L.o_sid_c = take(nc * 4);
  L.o_gt = take(nr * 4);
  L.o_tie = take(nr * 4);
  L.o_gpos = take((nr + 1) * 4);
  L.o_tpos = take((nr + 1) * 4);
  L.o_soff = take((R + 1) * 4);
  L.o_skeys = take(L.stored ? L.stair * 4 : 0);
  L.o_hist = take(256 * 4);
  L.o_misc = take(64 * 4);
  L.total = o;
  return L;
}

// Bitonic sort, descending, of n = 256 * PER keys in shared memory by the CTA's 256 threads.
// Warp w owns the block [w B, (w + 1) B), B = 32 PER, one key per lane in each of PER
// slots. Stages whose partner lies in the same block run in registers (partner j < 32
// lanes away: a shuffle; j >= 32: another slot of the same lane); only the stages with
// j >= B exchange through shared memory. Every thread calls.
template <int PER>
__device__ __forceinline__ void reg_stage(uint64_t (&v)[PER], int base, int k, int j) {
  const int lane = threadIdx.x & 31;
  if (j >= 32) {
    const int js = j >> 5;
#pragma unroll
    for (int sl = 0; sl < PER; ++sl) {
      if ((sl & js) == 0) {
        const int i = base + sl * 32 + lane;
        const bool desc = (i & k) == 0;
        const uint64_t x = v[sl], y = v[sl | js];
        if (desc ? (x < y) : (x > y)) {
          v[sl] = y;
          v[sl | js] = x;
        }
      }
    }
  } else {
    const bool lower = (lane & j) == 0;
#pragma unroll
    for (int sl = 0; sl < PER; ++sl) {
      const int i = base + sl * 32 + lane;
      const bool desc = (i & k) == 0;
      const uint64_t y = __shfl_xor_sync(0xffffffffu, v[sl], j);
      const bool keep_max = lower == desc;
      v[sl] = keep_max ? (v[sl] > y ? v[sl] : y) : (v[sl] < y ? v[sl] : y);
    }
  }
}

template <int PER>
__device__ void bitonic_desc_t(uint64_t* a) {
  constexpr int B = 32 * PER, n = 8 * B;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int base = warp * B;
  uint64_t v[PER];
#pragma unroll
  for (int sl = 0; sl < PER; ++sl) v[sl] = a[base + sl * 32 + lane];
#pragma unroll
  for (int k = 2; k <= B; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) reg_stage<PER>(v, base, k, j);
#pragma unroll
  for (int sl = 0; sl < PER; ++sl) a[base + sl * 32 + lane] = v[sl];
  __syncthreads();
  for (int k = 2 * B; k <= n; k <<= 1) {
    for (int j = k >> 1; j >= B; j >>= 1) {
      for (int p = threadIdx.x; p < (n >> 1); p += blockDim.x) {
        const int i = ((p & ~(j - 1)) << 1) | (p & (j - 1));
        const int l = i + j;
        const bool desc = (i & k) == 0;
        const uint64_t x = a[i], y = a[l];
        if (desc ? (x < y) : (x > y)) {
          a[i] = y;
          a[l] = x;
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int sl = 0; sl < PER; ++sl) v[sl] = a[base + sl * 32 + lane];
#pragma unroll
    for (int j = B >> 1; j > 0; j >>= 1) reg_stage<PER>(v, base, k, j);
#pragma unroll
    for (int sl = 0; sl < PER; ++sl) a[base + sl * 32 + lane] = v[sl];
    __syncthreads();
  }
}

// n is a power of two from 256 to 4096.
__device__ void bitonic_desc(uint64_t* a, int n) {
  switch (n >> 8) {
    case 1: bitonic_desc_t<1>(a); break;
    case 2: bitonic_desc_t<2>(a); break;
    case 4: bitonic_desc_t<4>(a); break;
    case 8: bitonic_desc_t<8>(a); break;
    default: bitonic_desc_t<16>(a); break;
  }
}

// Exclusive scans of two int arrays of length n <= 4 * blockDim.x, in place; returns the
// totals through `tot` (shared). Every thread calls.
__device__ void block_exscan2(const int* in0, const int* in1, int* out0, int* out1, int n, int* wsum,
                              int* tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int v0[4], v1[4], s0 = 0, s1 = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = tid * 4 + q;
    v0[q] = i < n ? in0[i] : 0;
    v1[q] = i < n ? in1[i] : 0;
    s0 += v0[q];
    s1 += v1[q];
  }
  int i0 = s0, i1 = s1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, i0, o), b = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) {
      i0 += a;
      i1 += b;
    }
  }
  if (lane == 31) {
    wsum[warp] = i0;
    wsum[32 + warp] = i1;
  }
  __syncthreads();
  if (tid == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      const int x = wsum[w], y = wsum[32 + w];
      wsum[w] = a;
      wsum[32 + w] = b;
      a += x;
      b += y;
    }
    tot[0] = a;
    tot[1] = b;
  }
  __syncthreads();
  int e0 = wsum[warp] + i0 - s0, e1 = wsum[32 + warp] + i1 - s1;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = tid * 4 + q;
    if (i < n) {
      out0[i] = e0;
      out1[i] = e1;
    }
    e0 += v0[q];
    e1 += v1[q];
  }
  __syncthreads();
}

// Deterministic block sum (fixed order): every thread calls; the result is returned to all.
__device__ float block_sum(float v, float* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
    red[32] = s;
  }
  __syncthreads();
  const float s = red[32];
  __syncthreads();
  return s;
}

// Warp 0 finds the radix digit: scanning digits from the top (DESC) or bottom, the digit b
// at which the running count first reaches `need`; returns b and the count before it.
__device__ void pick_digit(const int* hist, int need, bool desc, int* out_digit, int* out_before) {
  const int lane = threadIdx.x & 31;
  int cnt[8], sum = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int rank = lane * 8 + q;
    cnt[q] = hist[desc ? 255 - rank : rank];
    sum += cnt[q];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int excl = incl - sum;
  const unsigned bal = __ballot_sync(0xffffffffu, excl < need && need <= incl);
  if (bal != 0 && lane == __ffs(bal) - 1) {
    int acc = excl, q = 0;
    for (; q < 7; ++q) {
      if (acc + cnt[q] >= need) break;
      acc += cnt[q];
    }
    const int rank = lane * 8 + q;
    *out_digit = desc ? 255 - rank : rank;
    *out_before = acc;
  }
}

// Adds the lanes' votes to a shared histogram with one atomic per distinct bin of the warp
// (pair sums of one token fall into few bins, so per-lane atomics would serialise). Every
// lane of the warp calls it (uniform control flow).
__device__ __forceinline__ void hist_add_warp(int* hist, bool pred, uint32_t bin) {
  const uint32_t key = pred ? bin : 0xFFFFFFFFu;
  const unsigned peers = __match_any_sync(0xffffffffu, key);
  if (pred && (threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1))
    atomicAdd(&hist[bin], __popc(peers));
}

struct TopkArgs {
  const float* logits;  // [T, nr + nc]
  int32_t* ids;         // [T, K]
  float* w;             // [T, K]
  int T, nr, nc, K, renorm;
  unsigned* status;
  int32_t* counts;  // [N] or NULL: tasks per expert, counted as the ids are written
  TopkSmem L;
};

__global__ void __launch_bounds__(TK_THREADS) omni_topk_kernel(const TopkArgs g) {
  extern __shared__ __align__(16) uint8_t sm[];
  const TopkSmem& L = g.L;
  uint64_t* rk = (uint64_t*)(sm + L.o_rk);
  uint64_t* ck = (uint64_t*)(sm + L.o_ck);
  uint64_t* sel = (uint64_t*)(sm + L.o_sel);
  float* raw_r = (float*)(sm + L.o_raw_r);
  float* raw_c = (float*)(sm + L.o_raw_c);
  float* sv_r = (float*)(sm + L.o_sv_r);
  float* sv_c = (float*)(sm + L.o_sv_c);
  int* sid_r = (int*)(sm + L.o_sid_r);
  int* sid_c = (int*)(sm + L.o_sid_c);
  int* s_gt = (int*)(sm + L.o_gt);
  int* s_tie = (int*)(sm + L.o_tie);
  int* gpos = (int*)(sm + L.o_gpos);
  int* tpos = (int*)(sm + L.o_tpos);
  int* soff = (int*)(sm + L.o_soff);
  uint32_t* skeys = (uint32_t*)(sm + L.o_skeys);
  int* hist = (int*)(sm + L.o_hist);
  int* misc = (int*)(sm + L.o_misc);  // [0..63]: scan partials, totals, digits, counters
  float* red = (float*)(sm + L.o_hist);  // reused after the selection

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nr = g.nr, nc = g.nc, K = g.K, P = nr + nc;
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (t >= g.T) return;

  // 1. both axes: raw values and sort keys (padding keys 0 sort last)
  const float* lg = g.logits + (size_t)t * P;
  for (int i = tid; i < L.PP; i += TK_THREADS) {
    if (i < nr) {
      const float v = lg[i];
      raw_r[i] = v;
      rk[i] = composite(ord_key(v), (uint32_t)i);
    } else {
      rk[i] = 0;
    }
    if (i < nc) {
      const float v = lg[nr + i];
      raw_c[i] = v;
      ck[i] = composite(ord_key(v), (uint32_t)i);
    } else {
      ck[i] = 0;
    }
  }
  __syncthreads();
  bitonic_desc(rk, L.PP);
  bitonic_desc(ck, L.PP);
  for (int i = tid; i < nr; i += TK_THREADS) {
    const int id = (int)(0xFFFFFFFFu - (uint32_t)rk[i]);
    sid_r[i] = id;
    sv_r[i] = raw_r[id];
  }
  for (int i = tid; i < nc; i += TK_THREADS) {
    const int id = (int)(0xFFFFFFFFu - (uint32_t)ck[i]);
    sid_c[i] = id;
    sv_c[i] = raw_c[id];
  }
  __syncthreads();

  // 2. threshold key: the K-th largest pair-sum key over the staircase of sorted ranks
  const int R = min(nr, K);
  if (L.stored) {  // the staircase's keys, flattened row after row, in shared memory
    for (int r = tid; r < R; r += TK_THREADS) s_gt[r] = min(nc, K / (r + 1));
    __syncthreads();
    block_exscan2(s_gt, s_gt, soff, s_tie, R, misc, misc + 48);
    if (tid == 0) soff[R] = L.stair;
    __syncthreads();
    const int per = (L.stair + TK_THREADS - 1) / TK_THREADS;
    int f = tid * per;
    const int f1 = min(L.stair, f + per);
    if (f < f1) {
      int lo = 0, hi = R - 1;  // the row of f: last r with soff[r] <= f (rows are not empty)
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (soff[mid] <= f) lo = mid;
        else hi = mid - 1;
      }
      int r = lo, c = f - soff[lo], rend = soff[lo + 1];
      float a = sv_r[r];
      for (; f < f1; ++f, ++c) {
        if (f == rend) {
          ++r;
          c = 0;
          rend = soff[r + 1];
          a = sv_r[r];
        }
        skeys[f] = ord_key(a + sv_c[c]);
      }
    }
  }
  uint32_t prefix = 0, pmask = 0;
  int need = K;
  if (tid == 0) {
    misc[40] = 0;
    misc[41] = 0;
  }
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += TK_THREADS) hist[i] = 0;
    __syncthreads();
    if (L.stored) {
      for (int f = tid; f < L.stair; f += TK_THREADS) {
        const uint32_t key = skeys[f];
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
      }
    } else {
      for (int r = warp; r < R; r += TK_WARPS) {
        const int Lr = min(nc, K / (r + 1));
        const float a = sv_r[r];
        for (int c = lane; c < Lr; c += 32) {
          const uint32_t key = ord_key(a + sv_c[c]);
          if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
        }
      }
    }
    __syncthreads();
    if (warp == 0) pick_digit(hist, need, true, &misc[40], &misc[41]);
    __syncthreads();
    prefix |= (uint32_t)misc[40] << shift;
    pmask |= 0xFFu << shift;
    need -= misc[41];
    __syncthreads();
  }
  const uint32_t theta = prefix;

  // 3. per row of the whole grid: pairs above the threshold and pairs equal to it
  for (int r = tid; r < nr; r += TK_THREADS) {
    const float a = sv_r[r];
    int lo = 0, hi = nc;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (ord_key(a + sv_c[mid]) > theta) lo = mid + 1;
      else hi = mid;
    }
    const int gt = lo;
    hi = nc;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (ord_key(a + sv_c[mid]) >= theta) lo = mid + 1;
      else hi = mid;
    }
    s_gt[r] = gt;
    s_tie[r] = lo - gt;
  }
  __syncthreads();
  block_exscan2(s_gt, s_tie, gpos, tpos, nr, misc, misc + 48);
  const int gt_total = misc[48], tie_total = misc[49];
  const int take = K - gt_total;  // pairs taken at the threshold, 1 <= take <= tie_total
  if (tid == 0) {
    gpos[nr] = gt_total;
    tpos[nr] = tie_total;
  }

  // 4. the winners: every pair above the threshold, then the `take` lowest ids at it; one
  // thread per output slot finds its row by a binary search over the row offsets
  for (int i = tid; i < L.KP; i += TK_THREADS) sel[i] = 0;
  __syncthreads();
  for (int k = tid; k < min(gt_total, K); k += TK_THREADS) {
    int lo = 0, hi = nr - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (gpos[mid] <= k) lo = mid;
      else hi = mid - 1;
    }
    const int c = k - gpos[lo];
    sel[k] = composite(ord_key(sv_r[lo] + sv_c[c]), (uint32_t)sid_r[lo] * (uint32_t)nc + (uint32_t)sid_c[c]);
  }
  if (take == tie_total) {
    for (int k = tid; k < tie_total; k += TK_THREADS) {
      int lo = 0, hi = nr - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tpos[mid] <= k) lo = mid;
        else hi = mid - 1;
      }
      const int c = s_gt[lo] + (k - tpos[lo]);
      if (gt_total + k < K)
        sel[gt_total + k] = composite(theta, (uint32_t)sid_r[lo] * (uint32_t)nc + (uint32_t)sid_c[c]);
    }
  } else {
    // radix select (ascending) of the take-th smallest id among the pairs at the threshold
    uint32_t ipre = 0, imask = 0;
    int ineed = take;
    for (int shift = 16; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += TK_THREADS) hist[i] = 0;
      __syncthreads();
      for (int r = warp; r < nr; r += TK_WARPS) {
        const uint32_t rid = (uint32_t)sid_r[r] * (uint32_t)nc;
        const int c0 = s_gt[r];
        const int nt = s_tie[r];
        for (int cb = 0; cb < nt; cb += 32) {
          const int c = cb + lane;
          const uint32_t id = c < nt ? rid + (uint32_t)sid_c[c0 + c] : 0u;
          hist_add_warp(hist, c < nt && (id & imask) == ipre, (id >> shift) & 255);
        }
      }
      __syncthreads();
      if (warp == 0) pick_digit(hist, ineed, false, &misc[40], &misc[41]);
      __syncthreads();
      ipre |= (uint32_t)misc[40] << shift;
      imask |= 0xFFu << shift;
      ineed -= misc[41];
      __syncthreads();
    }
    if (tid == 0) misc[42] = 0;
    __syncthreads();
    for (int r = warp; r < nr; r += TK_WARPS) {
      const uint32_t rid = (uint32_t)sid_r[r] * (uint32_t)nc;
      const int c0 = s_gt[r];
      for (int c = lane; c < s_tie[r]; c += 32) {
        const uint32_t id = rid + (uint32_t)sid_c[c0 + c];
        if (id <= ipre) {
          const int pos = gt_total + atomicAdd(&misc[42], 1);
          if (pos < K) sel[pos] = composite(theta, id);
        }
      }
    }
  }
  __syncthreads();
  bitonic_desc(sel, L.KP);
  // every slot below K holds a pair unless the logits held a NaN: such a slot decodes to
  // expert 0 and the fault is reported
  const uint32_t N = (uint32_t)nr * (uint32_t)nc;
  auto decode = [&](uint64_t cv) -> uint32_t {
    const uint32_t id = 0xFFFFFFFFu - (uint32_t)cv;
    if (id >= N) {
      report(g.status, MOE_ERR_DEVICE_INDEX);
      return 0u;
    }
    return id;
  };

  // 5. weights and outputs
  float part = 0.f;
  float mr = 0.f, mc = 0.f, zr = 1.f, zc = 1.f, v0 = 0.f;
  if (g.renorm) {
    const uint32_t id0 = decode(sel[0]);
    v0 = raw_r[id0 / nc] + raw_c[id0 % nc];
    for (int k = tid; k < K; k += TK_THREADS) {
      const uint32_t id = decode(sel[k]);
      part += expf(raw_r[id / nc] + raw_c[id % nc] - v0);
    }
    zr = block_sum(part, red);
  } else {
    mr = sv_r[0];
    mc = sv_c[0];
    for (int i = tid; i < nr; i += TK_THREADS) part += expf(raw_r[i] - mr);
    zr = block_sum(part, red);
    part = 0.f;
    for (int i = tid; i < nc; i += TK_THREADS) part += expf(raw_c[i] - mc);
    zc = block_sum(part, red);
  }
  for (int k = tid; k < K; k += TK_THREADS) {
    const uint32_t id = decode(sel[k]);
    const float a = raw_r[id / nc], b = raw_c[id % nc];
    float w;
    if (g.renorm) w = expf(a + b - v0) / zr;
    else w = (expf(a - mr) / zr) * (expf(b - mc) / zc);
    g.ids[(size_t)t * K + k] = (int32_t)id;
    if (g.counts != nullptr) atomicAdd(&g.counts[id], 1);
    g.w[(size_t)t * K + k] = w;
  }
}

// ------------------------------------------------------------------ schedule
__global__ void omni_zero_kernel(int32_t* a, int32_t* b, long long n, int32_t* c) {
  pdl_wait();
  pdl_trigger();
  const long long i0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  for (long long i = i0; i < n; i += (long long)gridDim.x * blockDim.x) {
    a[i] = 0;
    b[i] = 0;
  }
  if (i0 == 0) *c = 0;
}

__global__ void omni_count_kernel(const int32_t* ids, long long M, int N, int32_t* counts,
                                  unsigned* status) {
  pdl_wait();
  pdl_trigger();
  for (long long a = blockIdx.x * (long long)blockDim.x + threadIdx.x; a < M;
       a += (long long)gridDim.x * blockDim.x) {
    const int e = ids[a];
    if ((unsigned)e >= (unsigned)N) {
      report(status, MOE_ERR_DEVICE_INDEX);
      continue;
    }
    atomicAdd(&counts[e], 1);
  }
}

constexpr int kScanTile = 4096;  // counts per CTA of the offsets scan: 1024 threads x 4

// Block-wide inclusive scan of one int per thread (1024 threads); returns the inclusive
// value and leaves the block total in *total.
__device__ int block_incl_scan(int v, int* ws, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += u;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int wv = ws[lane];
    int y = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += u;
    }
    ws[lane] = y - wv;
    if (lane == 31) *total = y;
  }
  __syncthreads();
  return x + ws[warp];
}

// Pass 1: the count total of each 4096-expert tile.
__global__ void __launch_bounds__(1024) omni_scan_sums_kernel(const int32_t* counts, int N,
                                                              int32_t* sums) {
  __shared__ int ws[32];
  __shared__ int total;
  pdl_wait();
  pdl_trigger();
  const int base = blockIdx.x * kScanTile + threadIdx.x * 4;
  int v = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (base + q < N) v += counts[base + q];
  block_incl_scan(v, ws, &total);
  if (threadIdx.x == 0) sums[blockIdx.x] = total;
}

// Pass 2: offsets = exclusive scan of counts; each tile adds the totals of the tiles before
// it (at most 256 of them); the last tile writes offsets[N].
__global__ void __launch_bounds__(1024) omni_scan_write_kernel(const int32_t* counts, int N,
                                                               const int32_t* sums,
                                                               int32_t* offsets) {
  __shared__ int ws[32];
  __shared__ int total, carry;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    int c = 0;
    for (int i = lane; i < (int)blockIdx.x; i += 32) c += sums[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) carry = c;
  }
  const int base = blockIdx.x * kScanTile + threadIdx.x * 4;
  int v[4], sum = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    v[q] = base + q < N ? counts[base + q] : 0;
    sum += v[q];
  }
  int run = block_incl_scan(sum, ws, &total) - sum + carry;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (base + q < N) offsets[base + q] = run;
    run += v[q];
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) offsets[N] = carry + total;
}

__global__ void omni_scatter_kernel(const int32_t* ids, long long M, int N, const int32_t* offsets,
                                    int32_t* cursor, int32_t* tmp) {
  pdl_wait();
  pdl_trigger();
  for (long long a = blockIdx.x * (long long)blockDim.x + threadIdx.x; a < M;
       a += (long long)gridDim.x * blockDim.x) {
    const int e = ids[a];
    if ((unsigned)e >= (unsigned)N) continue;
    tmp[offsets[e] + atomicAdd(&cursor[e], 1)] = (int32_t)a;
  }
}

constexpr int kWarpSortMax = 64;      // segments sorted inside one warp
constexpr int kBlockSortMax = 16384;  // segments sorted in one CTA's shared memory

// A warp per expert: segments of up to 64 slots are ranked in registers; longer ones are
// queued for omni_bigsort.
__global__ void omni_segsort_kernel(const int32_t* offsets, int N, const int32_t* tmp, int32_t* p2a,
                                    int32_t* a2p, int32_t* big_list, int32_t* big_count) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; e < N; e += nw) {
    const int off = offsets[e], n = offsets[e + 1] - off;
    if (n == 0) continue;
    if (n > kWarpSortMax) {
      if (lane == 0) big_list[atomicAdd(big_count, 1)] = e;
      continue;
    }
    const int v0 = lane < n ? tmp[off + lane] : 0x7fffffff;
    const int v1 = lane + 32 < n ? tmp[off + lane + 32] : 0x7fffffff;
    int r0 = 0, r1 = 0;
    for (int j = 0; j < 32; ++j) {
      const int u0 = __shfl_sync(0xffffffffu, v0, j), u1 = __shfl_sync(0xffffffffu, v1, j);
      r0 += (u0 < v0) + (u1 < v0);
      r1 += (u0 < v1) + (u1 < v1);
    }
    if (lane < n) {
      p2a[off + r0] = v0;
      a2p[v0] = off + r0;
    }
    if (lane + 32 < n) {
      p2a[off + r1] = v1;
      a2p[v1] = off + r1;
    }
  }
}

// One CTA per queued expert: a bitonic sort in shared memory for up to 16384 slots; beyond
// that, the expert's assignments are compacted in order straight from the ids.
__global__ void __launch_bounds__(1024) omni_bigsort_kernel(const int32_t* offsets, const int32_t* ids,
                                                            long long M, const int32_t* tmp,
                                                            int32_t* p2a, int32_t* a2p,
                                                            const int32_t* big_list,
                                                            const int32_t* big_count) {
  extern __shared__ int32_t vals[];  // kBlockSortMax
  __shared__ int wsum[33];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nbig = *big_count;
  for (int q = blockIdx.x; q < nbig; q += gridDim.x) {
    const int e = big_list[q];
    const int off = offsets[e], n = offsets[e + 1] - off;
    if (n <= kBlockSortMax) {
      const int np = pow2_at_least(n);
      for (int i = tid; i < np; i += blockDim.x) vals[i] = i < n ? tmp[off + i] : 0x7fffffff;
      __syncthreads();
      for (int k = 2; k <= np; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
          for (int p = tid; p < (np >> 1); p += blockDim.x) {
            const int i = ((p & ~(j - 1)) << 1) | (p & (j - 1));
            const int l = i + j;
            const bool asc = (i & k) == 0;
            const int x = vals[i], y = vals[l];
            if (asc ? (x > y) : (x < y)) {
              vals[i] = y;
              vals[l] = x;
            }
          }
          __syncthreads();
        }
      }
      for (int i = tid; i < n; i += blockDim.x) {
        p2a[off + i] = vals[i];
        a2p[vals[i]] = off + i;
      }
      __syncthreads();
    } else {
      int run = 0;
      for (long long base = 0; base < M; base += blockDim.x) {
        const long long a = base + tid;
        const int f = (a < M && ids[a] == e) ? 1 : 0;
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        if (lane == 0) wsum[warp] = __popc(bal);
        __syncthreads();
        if (tid == 0) {
          int s = 0;
          for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const int c = wsum[w];
            wsum[w] = s;
            s += c;
          }
          wsum[32] = s;
        }
        __syncthreads();
        if (f) {
          const int p = off + run + wsum[warp] + __popc(bal & lanemask_lt());
          p2a[p] = (int32_t)a;
          a2p[a] = p;
        }
        run += wsum[32];
        __syncthreads();
      }
    }
  }
}

// ------------------------------------------------------------------ experts
__device__ __forceinline__ uint4 ldg_nc(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds16(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Shared memory of one warp in the row-streaming kernels: R rows of d bf16 (CH 16-byte
// vectors per lane).
template <int CH, int R>
struct RowRing {
  static constexpr int ROW = CH * 32 * 16;
  static constexpr int BYTES = R * ROW;
};

// acc + (x.lo * w.lo) + (x.hi * w.hi) for two packed bf16 pairs, fp32 accumulation: the
// mixed-precision FMA takes the bf16 halves directly (a bf16 product is exact in fp32).
__device__ __forceinline__ float fma_bf16x2(uint32_t x, uint32_t w, float acc) {
  asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
      "mov.b32 {xl, xh}, %1;\n\tmov.b32 {wl, wh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, xl, wl, %0;\n\tfma.rn.f32.bf16 %0, xh, wh, %0;\n\t}"
      : "+f"(acc)
      : "r"(x), "r"(w));
  return acc;
}

// acc.{x, y} += {w.lo, w.hi} * hh.{x, y}: a packed bf16 pair widened to fp32 and one
// two-lane fp32 FMA.
__device__ __forceinline__ void fma2_bf16(uint32_t w, uint64_t hh, uint64_t& acc) {
  asm("{\n\t.reg .b32 lo, hi;\n\t.reg .b64 v;\n\t"
      "shl.b32 lo, %1, 16;\n\tand.b32 hi, %1, 0xffff0000;\n\t"
      "mov.b64 v, {lo, hi};\n\tfma.rn.f32x2 %0, v, %2, %0;\n\t}"
      : "+l"(acc)
      : "r"(w), "l"(hh));
}

// Sums v[i] over the 32 lanes for all NB values at once: a butterfly that halves the values
// held at each step (lane masks 16, 8, ...), then plain sums over the lane bits left; lane l
// returns the sum of v[l / (32 / NB)]. NB = 8: 9 shuffles for 8 sums.
template <int NB>
__device__ __forceinline__ float transpose_reduce(float (&v)[NB]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int half = NB / 2, sft = 16; half >= 1; half >>= 1, sft >>= 1) {
    const bool upper = (lane & sft) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
    }
  }
  float s = v[0];
#pragma unroll
  for (int sft = 32 / NB / 2; sft >= 1; sft >>= 1) s += __shfl_xor_sync(0xffffffffu, s, sft);
  return s;
}

// Expert-centric scalars. The expert-major task list is cut into equal contiguous ranges,
// one per warp. A warp keeps the current expert's w_in row in registers (loaded once per
// expert it meets) and streams its tasks' token rows from L2 through an R-deep cp.async
// ring in shared memory; each lane copies and later reads only its own 16-byte columns,
// so the ring needs no synchronisation beyond the lane's own cp.async groups. Tasks go in
// batches of 8: each lane keeps 8 partial dot products, one transposed reduction gives
// lanes 4i .. 4i + 3 the dot product of task i, and lane 4i writes that task's scalar
// h[a] = topk_w[a] * silu(x_{a / K} . w_in[e]). (Batches of 32, one task a lane, kept the
// unrolled loop too large for the instruction cache: no-instruction stalls led the warp
// state profile.)
template <int CH, int R>
__global__ void __launch_bounds__(256) omni_act_kernel(const bf16* __restrict__ x,
                                                       const bf16* __restrict__ w_in,
                                                       const int32_t* __restrict__ offsets,
                                                       const int32_t* __restrict__ p2a,
                                                       const float* __restrict__ topk_w,
                                                       float* __restrict__ h, int N, int K, int d,
                                                       int M, unsigned* status) {
  using Ring = RowRing<CH, R>;
  extern __shared__ __align__(16) uint8_t sm_act[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, wpc = blockDim.x >> 5;
  const uint32_t rbase = saddr(sm_act + (size_t)warp * Ring::BYTES);
  pdl_wait();
  pdl_trigger();
  const long long nw = (long long)gridDim.x * wpc, gw = (long long)blockIdx.x * wpc + warp;
  const long long per = (((long long)M + nw - 1) / nw + 31) & ~31LL;
  const int P0 = (int)min((long long)M, gw * per), P1 = (int)min((long long)M, gw * per + per);
  if (P0 >= P1) return;
  if (offsets[N] != M) {  // the schedule must cover every task
    if (lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
    return;
  }
  int lo = 0, hi = N - 1;  // the expert owning slot P0: last e with offsets[e] <= P0
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= P0) lo = mid;
    else hi = mid - 1;
  }
  int e = lo, e_end = offsets[e + 1];
  uint4 wv[CH];
  {
    const uint4* wr = reinterpret_cast<const uint4*>(w_in + (size_t)e * d);
#pragma unroll
    for (int j = 0; j < CH; ++j) wv[j] = ldg_nc(wr + lane + 32 * j);
  }
  // issue side: lane l holds the token of task ibase + l (-1: none or invalid)
  int ibase = P0 - 32, itok = -1;
  auto issue = [&](int q) {
    if (q < P1) {
      if (q >= ibase + 32) {
        ibase = q;
        const int a = q + lane < P1 ? p2a[q + lane] : -1;
        itok = (unsigned)a < (unsigned)M ? a / K : -1;
      }
      const int t = __shfl_sync(0xffffffffu, itok, q - ibase);
      if (t >= 0) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(x + (size_t)t * d);
        const uint32_t dst = rbase + ((q - P0) % R) * Ring::ROW;
#pragma unroll
        for (int j = 0; j < CH; ++j) cp_async16(dst + (lane + 32 * j) * 16, src + (lane + 32 * j) * 16);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < R; ++i) issue(P0 + i);
  constexpr int NB = 8;  // tasks a batch; lanes 4i .. 4i + 3 receive task i's sum
  for (int base = P0; base < P1; base += NB) {
    const int mine = base + (lane >> 2);
    int ca = (lane & 3) == 0 && mine < P1 ? p2a[mine] : -1;  // the task this lane writes
    if (ca >= M) {
      report(status, MOE_ERR_DEVICE_INDEX);
      ca = -1;
    }
    const float cw = ca >= 0 ? topk_w[ca] : 0.f;
    float v[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      const int p = base + i;
      float acc = 0.f;
      if (p < P1) {
        if (p >= e_end) {  // next expert with tasks
          while (p >= e_end && e < N - 1) {
            ++e;
            e_end = offsets[e + 1];
          }
          const uint4* wr = reinterpret_cast<const uint4*>(w_in + (size_t)e * d);
#pragma unroll
          for (int j = 0; j < CH; ++j) wv[j] = ldg_nc(wr + lane + 32 * j);
        }
        cp_async_wait<R - 1>();
        const uint32_t src = rbase + ((p - P0) % R) * Ring::ROW;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const uint4 xv = lds16(src + (lane + 32 * j) * 16);
          a0 = fma_bf16x2(xv.x, wv[j].x, a0);
          a1 = fma_bf16x2(xv.y, wv[j].y, a1);
          a0 = fma_bf16x2(xv.z, wv[j].z, a0);
          a1 = fma_bf16x2(xv.w, wv[j].w, a1);
        }
        acc = a0 + a1;
        issue(p + R);
      }
      v[i] = acc;
    }
    const float sdot = transpose_reduce<NB>(v);
    if (ca >= 0) h[ca] = cw * (sdot / (1.f + expf(-sdot)));
  }
  cp_async_wait<0>();
}

// Token-centric output. A CTA takes one token at a time; its WPT warps split the token's K
// tasks into contiguous chunks, stream the w_out rows through R-deep cp.async rings and keep
// 8 CH fp32 sums per lane; the warps' sums are then added in warp order (deterministic).
// One pass takes only the tasks whose expert lies in [elo, ehi) (a warp first compacts its
// chunk's (expert, scalar) pairs into shared memory): with the w_out table cut into slabs
// that fit in L2, each pass gathers its rows from L2 instead of DRAM. The first pass starts
// from zero, the others from the fp32 row y32[t] the previous one left; the last writes
// bf16 out[t], the others y32[t].
template <int CH, int R, int WPT>
__global__ void __launch_bounds__(WPT * 32) omni_out_kernel(const bf16* __restrict__ w_out,
                                                            const int32_t* __restrict__ ids,
                                                            const float* __restrict__ h,
                                                            bf16* __restrict__ out, float* y32,
                                                            int T, int K, int d, int N, int elo,
                                                            int ehi, int first, int last,
                                                            unsigned* status) {
  using Ring = RowRing<CH, R>;
  static_assert(Ring::BYTES >= CH * 32 * 8 * 4, "a warp's ring holds its partial row");
  extern __shared__ __align__(16) uint8_t sm_out[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int kc = (K + WPT - 1) / WPT;
  uint8_t* rg = sm_out + (size_t)warp * Ring::BYTES;
  const uint32_t rbase = saddr(rg);
  int2* list = reinterpret_cast<int2*>(sm_out + (size_t)WPT * Ring::BYTES) + (size_t)warp * kc;
  const unsigned lt = lanemask_lt();
  pdl_wait();
  pdl_trigger();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const int k0 = min(K, warp * kc), k1 = min(K, k0 + kc);
    const int32_t* tid_ = ids + (size_t)t * K;
    const float* th = h + (size_t)t * K;
    // this pass's tasks of the chunk, in k order
    int nv = 0;
    for (int q0 = k0; q0 < k1; q0 += 32) {
      const int q = q0 + lane;
      const int e = q < k1 ? tid_[q] : 0;
      const float hv = q < k1 ? th[q] : 0.f;
      if (q < k1 && (unsigned)e >= (unsigned)N) report(status, MOE_ERR_DEVICE_INDEX);
      const bool in = q < k1 && e >= elo && e < ehi;
      const unsigned b = __ballot_sync(0xffffffffu, in);
      if (in) list[nv + __popc(b & lt)] = make_int2(e, __float_as_int(hv));
      nv += __popc(b);
    }
    __syncwarp();
    uint64_t acc[CH][4];  // fp32 pairs (columns 2i, 2i + 1 of each 8-column chunk)
#pragma unroll
    for (int j = 0; j < CH; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[j][q] = 0ull;
    auto issue = [&](int i) {
      if (i < nv) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(w_out + (size_t)list[i].x * d);
        const int slot = i % R;
#pragma unroll
        for (int j = 0; j < CH; ++j)
          cp_async16(rbase + slot * Ring::ROW + (lane + 32 * j) * 16, src + (lane + 32 * j) * 16);
      }
      cp_async_commit();
    };
#pragma unroll
    for (int i = 0; i < R; ++i) issue(i);
    for (int i = 0; i < nv; ++i) {
      const float hv = __int_as_float(list[i].y);
      uint64_t hh;
      asm("mov.b64 %0, {%1, %1};" : "=l"(hh) : "f"(hv));
      cp_async_wait<R - 1>();
      const int slot = i % R;
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const uint4 v = lds16(rbase + slot * Ring::ROW + (lane + 32 * j) * 16);
        fma2_bf16(v.x, hh, acc[j][0]);
        fma2_bf16(v.y, hh, acc[j][1]);
        fma2_bf16(v.z, hh, acc[j][2]);
        fma2_bf16(v.w, hh, acc[j][3]);
      }
      issue(i + R);
    }
    cp_async_wait<0>();
    // this warp's partial row, [d] fp32, into its own (now idle) ring
    float* part = reinterpret_cast<float*>(rg);
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      uint4* dst = reinterpret_cast<uint4*>(part + (lane + 32 * j) * 8);
      dst[0] = make_uint4((uint32_t)acc[j][0], (uint32_t)(acc[j][0] >> 32), (uint32_t)acc[j][1],
                          (uint32_t)(acc[j][1] >> 32));
      dst[1] = make_uint4((uint32_t)acc[j][2], (uint32_t)(acc[j][2] >> 32), (uint32_t)acc[j][3],
                          (uint32_t)(acc[j][3] >> 32));
    }
    __syncthreads();
    for (int c8 = threadIdx.x; c8 < d / 8; c8 += WPT * 32) {
      float sum[8];
      float4* yrow = reinterpret_cast<float4*>(y32 + (size_t)t * d) + c8 * 2;
      if (first) {
#pragma unroll
        for (int q = 0; q < 8; ++q) sum[q] = 0.f;
      } else {
        const float4 y0 = yrow[0], y1 = yrow[1];
        sum[0] = y0.x;
        sum[1] = y0.y;
        sum[2] = y0.z;
        sum[3] = y0.w;
        sum[4] = y1.x;
        sum[5] = y1.y;
        sum[6] = y1.z;
        sum[7] = y1.w;
      }
#pragma unroll
      for (int w = 0; w < WPT; ++w) {
        const float4* src =
            reinterpret_cast<const float4*>(sm_out + (size_t)w * Ring::BYTES) + c8 * 2;
        const float4 x0 = src[0], x1 = src[1];
        sum[0] += x0.x;
        sum[1] += x0.y;
        sum[2] += x0.z;
        sum[3] += x0.w;
        sum[4] += x1.x;
        sum[5] += x1.y;
        sum[6] += x1.z;
        sum[7] += x1.w;
      }
      if (last) {
        *reinterpret_cast<uint4*>(out + (size_t)t * d + c8 * 8) = pack16(sum, bf16());
      } else {
        yrow[0] = make_float4(sum[0], sum[1], sum[2], sum[3]);
        yrow[1] = make_float4(sum[4], sum[5], sum[6], sum[7]);
      }
    }
    __syncthreads();
  }
}

// The page's output side (section 2.3: results added back per token by scatter-add), kept
// as a measured alternative to the token-centric gather: each warp owns an equal range of
// the expert-major task list, keeps the current expert's w_out row in registers and adds
// h[a] * w_out[e] into the token's fp32 row with vector reductions (red.global.add.v4.f32).
// The sum order is the order the reductions land in, so results vary in the last bits.
__global__ void omni_zero_f32_kernel(float4* __restrict__ y, long long n4) {
  pdl_wait();
  pdl_trigger();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x)
    y[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

__device__ __forceinline__ void red_add_v4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

template <int CH>
__global__ void __launch_bounds__(256) omni_scatter_out_kernel(const bf16* __restrict__ w_out,
                                                               const int32_t* __restrict__ offsets,
                                                               const int32_t* __restrict__ p2a,
                                                               const float* __restrict__ h,
                                                               float* __restrict__ y32, int N,
                                                               int K, int d, int M,
                                                               unsigned* status) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, wpc = blockDim.x >> 5;
  const long long nw = (long long)gridDim.x * wpc, gw = (long long)blockIdx.x * wpc + (threadIdx.x >> 5);
  const long long per = ((long long)M + nw - 1) / nw;
  const int P0 = (int)min((long long)M, gw * per), P1 = (int)min((long long)M, gw * per + per);
  if (P0 >= P1) return;
  if (offsets[N] != M) {
    if (lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
    return;
  }
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= P0) lo = mid;
    else hi = mid - 1;
  }
  int e = lo, e_end = offsets[e + 1];
  uint4 wv[CH];
  {
    const uint4* wr = reinterpret_cast<const uint4*>(w_out + (size_t)e * d);
#pragma unroll
    for (int j = 0; j < CH; ++j) wv[j] = ldg_nc(wr + lane + 32 * j);
  }
  for (int base = P0; base < P1; base += 32) {
    const int a = base + lane < P1 ? p2a[base + lane] : -1;
    const bool ok = (unsigned)a < (unsigned)M;
    const int tl = ok ? a / K : -1;
    const float hl = ok ? h[a] : 0.f;
    const int n = min(32, P1 - base);
    for (int i = 0; i < n; ++i) {
      const int p = base + i;
      if (p >= e_end) {
        while (p >= e_end && e < N - 1) {
          ++e;
          e_end = offsets[e + 1];
        }
        const uint4* wr = reinterpret_cast<const uint4*>(w_out + (size_t)e * d);
#pragma unroll
        for (int j = 0; j < CH; ++j) wv[j] = ldg_nc(wr + lane + 32 * j);
      }
      const int t = __shfl_sync(0xffffffffu, tl, i);
      const float hv = __shfl_sync(0xffffffffu, hl, i);
      if (t < 0) {
        if (lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
        continue;
      }
      float* row = y32 + (size_t)t * d;
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        float f[8];
        unpack16(wv[j], f, bf16());
        float* dst = row + (lane + 32 * j) * 8;
        red_add_v4(dst, hv * f[0], hv * f[1], hv * f[2], hv * f[3]);
        red_add_v4(dst + 4, hv * f[4], hv * f[5], hv * f[6], hv * f[7]);
      }
    }
  }
}

__global__ void omni_to_bf16_kernel(const float4* __restrict__ y32, uint2* __restrict__ out,
                                    long long n4) {
  pdl_wait();
  pdl_trigger();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 v = y32[i];
    out[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

// ------------------------------------------------------------------ host launchers
template <typename Kern>
bool set_smem(Kern k, int bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

int grid_cap(long long work, int threads, int per_sm) {
  const long long want = (work + threads - 1) / threads;
  const long long cap = (long long)sm_count() * per_sm;
  const long long g = want < cap ? want : cap;
  return (int)(g < 1 ? 1 : g);
}

template <int NT>
moe_status launch_logits_nt(const CUtensorMap& mx, const CUtensorMap& mr, const CUtensorMap& mc,
                            const LogitsArgs& a, int tiles, int ctiles, cudaStream_t st) {
  constexpr int STAGE = LA_BYTES + (NT / 64) * LB_CHUNK;
  const int smem = L_STAGES * STAGE + 1024 + 128;
  auto kern = omni_logits_kernel<NT>;
  if (!set_smem(kern, smem)) return MOE_ERR_CUDA;
  launch_begin(K_OMNI_LOGITS, st);
  launch_kernel(kern, dim3((unsigned)tiles, (unsigned)ctiles), dim3(L_THREADS), (size_t)smem, st, 1u,
                mx, mr, mc, a);
  return launch_end(K_OMNI_LOGITS, st);
}

int axis_tile(int n) {  // columns per tile for an axis of n: a multiple of 64, at most 256
  const int tiles = (n + 255) / 256;
  const int per = (n + tiles - 1) / tiles;
  return ((per + 63) / 64) * 64;
}

template <typename Kern>
int resident_ctas(Kern k, int threads, int smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem) != cudaSuccess || n < 1)
    n = 1;
  return n;
}

template <int CH, int R>
moe_status launch_act_ch(const moe_omni_shape& s, const void* x, const void* w_in,
                         const int32_t* offsets, const int32_t* p2a, const float* topk_w, float* h,
                         cudaStream_t st) {
  const int N = s.n_rows * s.n_cols;
  constexpr int BYTES = RowRing<CH, R>::BYTES;
  const int warps = max(1, min(8, (64 * 1024) / BYTES));
  const int smem = warps * BYTES;
  auto kern = omni_act_kernel<CH, R>;
  if (!set_smem(kern, smem)) return MOE_ERR_CUDA;
  const int grid = sm_count() * resident_ctas(kern, warps * 32, smem);
  launch_begin(K_OMNI_ACT, st);
  launch_kernel(kern, dim3((unsigned)grid), dim3(warps * 32), (size_t)smem, st, 1u, (const bf16*)x,
                (const bf16*)w_in, offsets, p2a, topk_w, h, N, s.K, s.d, s.T * s.K,
                device_status_ptr());
  return launch_end(K_OMNI_ACT, st);
}

// w_out bytes a slab of the output gather may hold (it then stays in L2 between the tokens
// that read it): a 105 MB half of a 210 MB table measured as fast as a table that fits.
constexpr size_t kSlabBytes = 112u << 20;

template <int CH, int R, int WPT>
moe_status launch_out_ch(const moe_omni_shape& s, const void* w_out, const int32_t* ids,
                         const float* h, void* out, float* y32, cudaStream_t st) {
  const int N = s.n_rows * s.n_cols;
  const int kc = (s.K + WPT - 1) / WPT;
  const int smem = WPT * (RowRing<CH, R>::BYTES + kc * 8);
  auto kern = omni_out_kernel<CH, R, WPT>;
  if (!set_smem(kern, smem)) return MOE_ERR_CUDA;
  const int cap = sm_count() * resident_ctas(kern, WPT * 32, smem);
  const int grid = s.T < cap ? s.T : cap;
  // slabs of the expert table when there is an fp32 row to carry the sums between them
  const size_t table = (size_t)N * s.d * 2;
  const int S = (y32 != nullptr && table > kSlabBytes) ? (int)((table + kSlabBytes - 1) / kSlabBytes)
                                                       : 1;
  for (int p = 0; p < S; ++p) {
    const int elo = (int)((long long)N * p / S), ehi = (int)((long long)N * (p + 1) / S);
    launch_begin(K_OMNI_OUT, st);
    launch_kernel(kern, dim3((unsigned)grid), dim3(WPT * 32), (size_t)smem, st, 1u,
                  (const bf16*)w_out, ids, h, (bf16*)out, y32, s.T, s.K, s.d, N, elo, ehi,
                  p == 0 ? 1 : 0, p == S - 1 ? 1 : 0, device_status_ptr());
    const moe_status r = launch_end(K_OMNI_OUT, st);
    if (r != MOE_OK) return r;
  }
  return MOE_OK;
}

}  // namespace

// ------------------------------------------------------------------ library-internal API
moe_status launch_omni_logits(const moe_omni_shape& s, const void* x, const void* w_row,
                              const void* w_col, float* logits, cudaStream_t st) {
  const int nt = max(axis_tile(s.n_rows), axis_tile(s.n_cols));
  const int ct_r = (s.n_rows + nt - 1) / nt, ct_c = (s.n_cols + nt - 1) / nt;
  const int tiles = (s.T + LBM - 1) / LBM;
  CUtensorMap mx, mr, mc;
  const uint64_t dx[2] = {(uint64_t)s.d, (uint64_t)s.T}, sx[1] = {(uint64_t)s.d * 2};
  const uint32_t bx[2] = {64, 128};
  const uint64_t dr[2] = {(uint64_t)s.n_rows, (uint64_t)s.d}, sr[1] = {(uint64_t)s.n_rows * 2};
  const uint64_t dc[2] = {(uint64_t)s.n_cols, (uint64_t)s.d}, sc[1] = {(uint64_t)s.n_cols * 2};
  const uint32_t bw[2] = {64, 64};
  if (!make_map(&mx, x, 2, dx, sx, bx) || !make_map(&mr, w_row, 2, dr, sr, bw) ||
      !make_map(&mc, w_col, 2, dc, sc, bw))
    return MOE_ERR_CUDA;
  LogitsArgs a;
  a.logits = logits;
  a.T = s.T;
  a.nr = s.n_rows;
  a.nc = s.n_cols;
  a.P = s.n_rows + s.n_cols;
  a.ct_r = ct_r;
  a.kblocks = s.d / LBK;
  a.status = device_status_ptr();
  a.limit_ns = kWaitLimitNs;
  switch (nt) {
    case 64: return launch_logits_nt<64>(mx, mr, mc, a, tiles, ct_r + ct_c, st);
    case 128: return launch_logits_nt<128>(mx, mr, mc, a, tiles, ct_r + ct_c, st);
    case 192: return launch_logits_nt<192>(mx, mr, mc, a, tiles, ct_r + ct_c, st);
    default: return launch_logits_nt<256>(mx, mr, mc, a, tiles, ct_r + ct_c, st);
  }
}

moe_status launch_omni_topk(const moe_omni_shape& s, const float* logits, int32_t* ids, float* w,
                            int32_t* counts, cudaStream_t st) {
  const TopkSmem L = topk_smem_layout(s.n_rows, s.n_cols, s.K);
  const int smem = L.total;
  if (!set_smem(omni_topk_kernel, smem)) return MOE_ERR_CUDA;
  TopkArgs a;
  a.logits = logits;
  a.ids = ids;
  a.w = w;
  a.T = s.T;
  a.nr = s.n_rows;
  a.nc = s.n_cols;
  a.K = s.K;
  a.renorm = s.renormalize;
  a.status = device_status_ptr();
  a.counts = counts;
  a.L = L;
  launch_begin(K_OMNI_TOPK, st);
  launch_kernel(omni_topk_kernel, dim3((unsigned)s.T), dim3(TK_THREADS), (size_t)smem, st, 1u, a);
  return launch_end(K_OMNI_TOPK, st);
}

// Scratch of the schedule: cursor [N], unsorted slots [T K], queued experts [N], queue length
// (64 ints), the scan's tile totals (256).
size_t omni_schedule_scratch_bytes(const moe_omni_shape& s) {
  const size_t N = (size_t)s.n_rows * s.n_cols, M = (size_t)s.T * s.K;
  return (N + M + N + 64 + 256) * 4;
}

// Zeroes the schedule's per-expert counts and cursors and its queue length.
moe_status launch_omni_zero(const moe_omni_shape& s, int32_t* counts, void* scratch,
                            cudaStream_t st) {
  const int N = s.n_rows * s.n_cols;
  const long long M = (long long)s.T * s.K;
  int32_t* cursor = (int32_t*)scratch;
  int32_t* big_count = cursor + N + M + N;
  launch_begin(K_OMNI_COUNT, st);
  launch_kernel(omni_zero_kernel, dim3((unsigned)grid_cap(N, 256, 4)), dim3(256), 0, st, 1u, counts,
                cursor, (long long)N, big_count);
  return launch_end(K_OMNI_COUNT, st);
}

// The task list grouped by expert. counted: counts were zeroed and filled already (by the
// top-K kernel). stable: each expert's slots sorted by assignment id (= token) and
// assign_to_perm written; otherwise the order inside an expert is the order the scatter
// claimed the slots in, and assign_to_perm is not written.
moe_status launch_omni_schedule(const moe_omni_shape& s, const int32_t* ids, int32_t* counts,
                                int32_t* offsets, int32_t* a2p, int32_t* p2a, void* scratch,
                                bool counted, bool stable, cudaStream_t st) {
  const int N = s.n_rows * s.n_cols;
  const long long M = (long long)s.T * s.K;
  int32_t* cursor = (int32_t*)scratch;
  int32_t* tmp = cursor + N;
  int32_t* big_list = tmp + M;
  int32_t* big_count = big_list + N;
  int32_t* scan_sums = big_count + 64;
  unsigned* status = device_status_ptr();
  moe_status r;
  if (!counted) {
    if ((r = launch_omni_zero(s, counts, scratch, st)) != MOE_OK) return r;
    launch_begin(K_OMNI_COUNT, st);
    launch_kernel(omni_count_kernel, dim3((unsigned)grid_cap(M, 256, 8)), dim3(256), 0, st, 1u, ids,
                  M, N, counts, status);
    if ((r = launch_end(K_OMNI_COUNT, st)) != MOE_OK) return r;
  }
  const int scan_tiles = (N + kScanTile - 1) / kScanTile;
  launch_begin(K_OMNI_SCAN, st);
  launch_kernel(omni_scan_sums_kernel, dim3((unsigned)scan_tiles), dim3(1024), 0, st, 1u,
                (const int32_t*)counts, N, scan_sums);
  if ((r = launch_end(K_OMNI_SCAN, st)) != MOE_OK) return r;
  launch_begin(K_OMNI_SCAN, st);
  launch_kernel(omni_scan_write_kernel, dim3((unsigned)scan_tiles), dim3(1024), 0, st, 1u,
                (const int32_t*)counts, N, (const int32_t*)scan_sums, offsets);
  if ((r = launch_end(K_OMNI_SCAN, st)) != MOE_OK) return r;
  launch_begin(K_OMNI_SCATTER, st);
  launch_kernel(omni_scatter_kernel, dim3((unsigned)grid_cap(M, 256, 8)), dim3(256), 0, st, 1u, ids,
                M, N, (const int32_t*)offsets, cursor, stable ? tmp : p2a);
  if ((r = launch_end(K_OMNI_SCATTER, st)) != MOE_OK) return r;
  if (!stable) return MOE_OK;
  launch_begin(K_OMNI_SORT, st);
  launch_kernel(omni_segsort_kernel, dim3((unsigned)grid_cap((long long)N * 32, 256, 8)), dim3(256), 0,
                st, 1u, (const int32_t*)offsets, N, (const int32_t*)tmp, p2a, a2p, big_list,
                big_count);
  if ((r = launch_end(K_OMNI_SORT, st)) != MOE_OK) return r;
  const int bsmem = kBlockSortMax * 4;
  if (!set_smem(omni_bigsort_kernel, bsmem)) return MOE_ERR_CUDA;
  launch_begin(K_OMNI_SORT, st);
  launch_kernel(omni_bigsort_kernel, dim3((unsigned)sm_count()), dim3(1024), (size_t)bsmem, st, 1u,
                (const int32_t*)offsets, ids, M, (const int32_t*)tmp, p2a, a2p,
                (const int32_t*)big_list, (const int32_t*)big_count);
  return launch_end(K_OMNI_SORT, st);
}

moe_status launch_omni_act(const moe_omni_shape& s, const void* x, const void* w_in,
                           const int32_t* offsets, const int32_t* p2a, const float* topk_w,
                           float* h, cudaStream_t st) {
  switch (s.d / 256) {
    case 1: return launch_act_ch<1, 8>(s, x, w_in, offsets, p2a, topk_w, h, st);
    case 2: return launch_act_ch<2, 6>(s, x, w_in, offsets, p2a, topk_w, h, st);
    case 3: return launch_act_ch<3, 4>(s, x, w_in, offsets, p2a, topk_w, h, st);
    case 4: return launch_act_ch<4, 3>(s, x, w_in, offsets, p2a, topk_w, h, st);
    case 5: return launch_act_ch<5, 4>(s, x, w_in, offsets, p2a, topk_w, h, st);
    case 6: return launch_act_ch<6, 2>(s, x, w_in, offsets, p2a, topk_w, h, st);
    case 7: return launch_act_ch<7, 2>(s, x, w_in, offsets, p2a, topk_w, h, st);
    case 8: return launch_act_ch<8, 2>(s, x, w_in, offsets, p2a, topk_w, h, st);
    default: return launch_act_ch<16, 2>(s, x, w_in, offsets, p2a, topk_w, h, st);
  }
}

moe_status launch_omni_out(const moe_omni_shape& s, const void* w_out, const int32_t* ids,
                           const float* h, void* out, float* y32, cudaStream_t st) {
  switch (s.d / 256) {
    case 1: return launch_out_ch<1, 8, 4>(s, w_out, ids, h, out, y32, st);
    case 2: return launch_out_ch<2, 6, 4>(s, w_out, ids, h, out, y32, st);
    case 3: return launch_out_ch<3, 4, 4>(s, w_out, ids, h, out, y32, st);
    case 4: return launch_out_ch<4, 4, 4>(s, w_out, ids, h, out, y32, st);
    case 5: return launch_out_ch<5, 4, 4>(s, w_out, ids, h, out, y32, st);
    case 6: return launch_out_ch<6, 2, 4>(s, w_out, ids, h, out, y32, st);
    case 7: return launch_out_ch<7, 2, 4>(s, w_out, ids, h, out, y32, st);
    case 8: return launch_out_ch<8, 2, 4>(s, w_out, ids, h, out, y32, st);
    default: return launch_out_ch<16, 2, 4>(s, w_out, ids, h, out, y32, st);
  }
}

moe_status launch_omni_out_scatter(const moe_omni_shape& s, const void* w_out,
                                   const int32_t* offsets, const int32_t* p2a, const float* h,
                                   float* y32, void* out, cudaStream_t st) {
  const int N = s.n_rows * s.n_cols;
  const long long n4 = (long long)s.T * s.d / 4;
  moe_status r;
  launch_begin(K_OMNI_OUT, st);
  launch_kernel(omni_zero_f32_kernel, dim3((unsigned)grid_cap(n4, 256, 8)), dim3(256), 0, st, 1u,
                (float4*)y32, n4);
  if ((r = launch_end(K_OMNI_OUT, st)) != MOE_OK) return r;
  const int grid = sm_count() * 8;
  launch_begin(K_OMNI_OUT, st);
  switch (s.d / 256) {
#define OMNI_SCATTER_CASE(C)                                                                      \
  case C:                                                                                         \
    launch_kernel(omni_scatter_out_kernel<C>, dim3((unsigned)grid), dim3(256), 0, st, 1u,         \
                  (const bf16*)w_out, offsets, p2a, h, y32, N, s.K, s.d, s.T * s.K,               \
                  device_status_ptr());                                                           \
    break;
    OMNI_SCATTER_CASE(1)
    OMNI_SCATTER_CASE(2)
    OMNI_SCATTER_CASE(3)
    OMNI_SCATTER_CASE(4)
    OMNI_SCATTER_CASE(5)
    OMNI_SCATTER_CASE(6)
    OMNI_SCATTER_CASE(7)
    OMNI_SCATTER_CASE(8)
    default:
      OMNI_SCATTER_CASE(16)
#undef OMNI_SCATTER_CASE
  }
  if ((r = launch_end(K_OMNI_OUT, st)) != MOE_OK) return r;
  launch_begin(K_OMNI_OUT, st);
  launch_kernel(omni_to_bf16_kernel, dim3((unsigned)grid_cap(n4, 256, 8)), dim3(256), 0, st, 1u,
                (const float4*)y32, (uint2*)out, n4);
  return launch_end(K_OMNI_OUT, st);
}

}  // namespace moe

// ------------------------------------------------------------------ C ABI
namespace moe {
namespace {

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

moe_status check_omni(const moe_omni_shape* s) {
  if (s == nullptr) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->n_rows < 1 || s->n_cols < 1 || s->K < 1 || s->d < 256 || s->d % 256 != 0)
    return MOE_ERR_INVALID_ARG;
  if (s->output_mode < 0 || s->output_mode > 1) return MOE_ERR_INVALID_ARG;
  const long long N = (long long)s->n_rows * s->n_cols;
  if (s->K > N) return MOE_ERR_INVALID_ARG;
  if (s->n_rows > 1024 || s->n_cols > 1024 || N > (1LL << 20) || s->K > 4096)
    return MOE_ERR_UNSUPPORTED;
  const int ch = s->d / 256;
  if (ch > 8 && ch != 16) return MOE_ERR_UNSUPPORTED;
  if ((long long)s->T * s->K > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

void omni_layout(const moe_omni_shape& s, moe_omni_layout* L) {
  const size_t T = (size_t)s.T, K = (size_t)s.K, M = T * K;
  const size_t N = (size_t)s.n_rows * s.n_cols, P = (size_t)s.n_rows + s.n_cols;
  size_t o = 0;
  L->logits = o;
  o = al256(o + T * P * 4);
  L->topk_ids = o;
  o = al256(o + M * 4);
  L->topk_w = o;
  o = al256(o + M * 4);
  L->counts = o;
  o = al256(o + N * 4);
  L->offsets = o;
  o = al256(o + (N + 1) * 4);
  L->assign_to_perm = o;
  o = al256(o + M * 4);
  L->perm_to_assign = o;
  o = al256(o + M * 4);
  L->h = o;
  o = al256(o + M * 4);
  L->scratch = o;
  o = al256(o + omni_schedule_scratch_bytes(s));
  L->y32 = o;
  o = al256(o + T * (size_t)s.d * 4);
  L->total = o;
}

bool al16(const void* p) { return ((uintptr_t)p & 15) == 0; }

moe_status omni_route_impl(const moe_omni_shape& s, const void* x, const void* w_row,
                           const void* w_col, const float* logits_in, float* logits_out,
                           int32_t* ids, float* w, int32_t* counts, cudaStream_t st) {
  const float* lg = logits_in;
  if (lg == nullptr) {
    if (!x || !w_row || !w_col || !logits_out) return MOE_ERR_INVALID_ARG;
    if (s.n_rows % 8 != 0 || s.n_cols % 8 != 0) return MOE_ERR_UNSUPPORTED;
    if (!al16(x) || !al16(w_row) || !al16(w_col) || !al16(logits_out)) return MOE_ERR_INVALID_ARG;
    const moe_status r = launch_omni_logits(s, x, w_row, w_col, logits_out, st);
    if (r != MOE_OK) return r;
    lg = logits_out;
  }
  return launch_omni_topk(s, lg, ids, w, counts, st);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_omni_workspace_size(const moe_omni_shape* s) {
  if (check_omni(s) != MOE_OK) return 0;
  moe_omni_layout L;
  omni_layout(*s, &L);
  return L.total;
}

moe_status moe_omni_workspace_layout(const moe_omni_shape* s, moe_omni_layout* L) {
  const moe_status r = check_omni(s);
  if (r != MOE_OK) return r;
  if (L == nullptr) return MOE_ERR_INVALID_ARG;
  omni_layout(*s, L);
  return MOE_OK;
}

moe_status moe_omni_route(const moe_omni_shape* s, const void* x, const void* w_row,
                          const void* w_col, const float* logits_in, float* logits_out,
                          int32_t* topk_ids, float* topk_w, moe_stream_t stream) {
  moe_status r = check_omni(s);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  return omni_route_impl(*s, x, w_row, w_col, logits_in, logits_out, topk_ids, topk_w, nullptr,
                         (cudaStream_t)stream);
}

moe_status moe_omni_schedule(const moe_omni_shape* s, const int32_t* topk_ids, int32_t* counts,
                             int32_t* offsets, int32_t* assign_to_perm, int32_t* perm_to_assign,
                             void* workspace, size_t ws_bytes, moe_stream_t stream) {
  moe_status r = check_omni(s);
  if (r != MOE_OK) return r;
  if (!counts || !offsets || (s->T > 0 && (!topk_ids || !assign_to_perm || !perm_to_assign)))
    return MOE_ERR_INVALID_ARG;
  moe_omni_layout L;
  omni_layout(*s, &L);
  if (workspace == nullptr || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  return launch_omni_schedule(*s, topk_ids, counts, offsets, assign_to_perm, perm_to_assign,
                              (uint8_t*)workspace + L.scratch, false, true, (cudaStream_t)stream);
}

moe_status moe_omni_experts(const moe_omni_shape* s, const void* x, const void* w_in,
                            const void* w_out, const int32_t* topk_ids, const float* topk_w,
                            const int32_t* offsets, const int32_t* perm_to_assign, float* h,
                            void* out, moe_stream_t stream) {
  moe_status r = check_omni(s);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!x || !w_in || !w_out || !topk_ids || !topk_w || !offsets || !perm_to_assign || !h || !out)
    return MOE_ERR_INVALID_ARG;
  if (!al16(x) || !al16(w_in) || !al16(w_out) || !al16(out)) return MOE_ERR_INVALID_ARG;
  const cudaStream_t st = (cudaStream_t)stream;
  if ((r = launch_omni_act(*s, x, w_in, offsets, perm_to_assign, topk_w, h, st)) != MOE_OK) return r;
  return launch_omni_out(*s, w_out, topk_ids, h, out, nullptr, st);  // no fp32 rows: one pass
}

moe_status moe_omni_forward(const moe_omni_shape* s, const void* x, const void* w_row,
                            const void* w_col, const float* logits_in, const void* w_in,
                            const void* w_out, void* out, void* workspace, size_t ws_bytes,
                            moe_stream_t stream) {
  moe_status r = check_omni(s);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!x || !w_in || !w_out || !out) return MOE_ERR_INVALID_ARG;
  moe_omni_layout L;
  omni_layout(*s, &L);
  if (workspace == nullptr || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!al16(workspace)) return MOE_ERR_INVALID_ARG;
  uint8_t* ws = (uint8_t*)workspace;
  float* logits = (float*)(ws + L.logits);
  int32_t* ids = (int32_t*)(ws + L.topk_ids);
  float* w = (float*)(ws + L.topk_w);
  int32_t* counts = (int32_t*)(ws + L.counts);
  int32_t* offsets = (int32_t*)(ws + L.offsets);
  int32_t* a2p = (int32_t*)(ws + L.assign_to_perm);
  int32_t* p2a = (int32_t*)(ws + L.perm_to_assign);
  float* h = (float*)(ws + L.h);
  const cudaStream_t st = (cudaStream_t)stream;
  // counts are zeroed first and filled by the top-K kernel; the experts need the tasks
  // grouped by expert only, so the order inside an expert is left as the scatter made it
  if ((r = launch_omni_zero(*s, counts, ws + L.scratch, st)) != MOE_OK) return r;
  if ((r = omni_route_impl(*s, x, w_row, w_col, logits_in, logits, ids, w, counts, st)) != MOE_OK)
    return r;
  if ((r = launch_omni_schedule(*s, ids, counts, offsets, a2p, p2a, ws + L.scratch, true, false,
                                st)) != MOE_OK)
    return r;
  if (!al16(x) || !al16(w_in) || !al16(w_out) || !al16(out)) return MOE_ERR_INVALID_ARG;
  if ((r = launch_omni_act(*s, x, w_in, offsets, p2a, w, h, st)) != MOE_OK) return r;
  if (s->output_mode == 0)  // gathered per token, in L2-sized slabs of w_out
    return launch_omni_out(*s, w_out, ids, h, out, (float*)(ws + L.y32), st);
  return launch_omni_out_scatter(*s, w_out, offsets, p2a, h, (float*)(ws + L.y32), out, st);
}

}  // extern "C"
