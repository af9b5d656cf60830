// Router on the tensor cores for bf16 shapes: logits = x W_r (+ bias) with tcgen05, then
// softmax and top-K in the epilogue, one token per thread.
//
// "How AI chips support MoE", chapter 4, section 4.2: the gate is a small dense linear map
// that every token passes through and that the experts wait on; section 4.3: top-K is a
// partial sort per token. "Two upstream innovations of MoE: Routing-Free and OmniMoE",
// section 1.1: Router -> Softmax -> TopK.
//
// The router GEMM (M = T tokens, N = E experts, K = d) has an arithmetic intensity of about
// E FLOP per byte of x, so at E >= 32 fp32 FMA units cannot keep up with HBM; tcgen05 can.
// Default layout: one tile of up to 128 tokens per cluster of S CTAs (S <= 8) that split
// the d contraction (k-blocks of 64); each accumulates its partial 128 x N tile in TMEM
// (N = E rounded up to 16, fp32) and copies it column-major into its shared memory. After
// a cluster barrier every rank finishes a contiguous share of the tile's rows, one thread
// per row, adding the partials of ranks 0..S-1 in that fixed order through distributed
// shared memory (deterministic, no atomics, no global scratch): + bias, optional logits
// store, register top-K by insertion (value descending, ties to the lower id, +0 == -0),
// softmax weights over the selected (renormalised) or over all E with an online sum. With
// S = 1 the CTA's 128 threads own one row each and stage the outputs for coalesced stores.
// On request (moe_set_route_layout(2)) every CTA owns one tile of ceil(T / SMs) <= 128
// tokens over the whole of d instead: no cluster; the x tile is loaded with exactly its own
// rows (the MMA still computes 128 rows; rows past the tile read whatever follows in shared
// memory and are never used, since a row of D depends on the same row of A only), so a
// stage holds ceil(rows/8) KB of x and the ring is as deep as shared memory allows. It is
// slower: the kernel is bound by issuing its small-N MMAs, and that form issues one per
// 16-wide k step for fewer useful rows.
// Roles per CTA (128 threads): warp 0 issues the TMA loads (x tile rows x 64 and the W_r
// tile 64 x N, 128-byte swizzle), warp 1 the MMAs (M=128, N, K=16, A K-major, B MN-major),
// both as warp-uniform loops with one elected lane issuing; then all four warps read TMEM
// (warp w owns lanes 32w..32w+31). Each tile starts its k-blocks at a different offset so
// that the CTAs do not all read the same W_r lines at once.
// Every mbarrier wait is bounded; on expiry the status word records MOE_ERR_TIMEOUT.
#include <math.h>

#include "common.cuh"

namespace moe {

extern int g_route_layout;  // 0 automatic (split), 1 split over clusters, 2 one tile per CTA

namespace {

constexpr int RBM = 128, RBK = 64;
constexpr int RA_BYTES = RBM * RBK * 2;  // 16 KB
constexpr int RB_CHUNK = RBK * 64 * 2;   // 8 KB: 64 k-rows x 64 experts
constexpr int R_THREADS = 128;
constexpr int KMAX = 8;

// Pipeline depth: the x stream is latency-bound per CTA, so small-N stages (24 KB) go 8 deep.
__host__ __device__ constexpr int route_stages(int N) { return N <= 64 ? 8 : (N <= 128 ? 6 : 4); }

struct RouteArgs {
  const float* bias;
  float* logits_out;
  int32_t* topk_ids;
  float* topk_w;
  int T, E, K, renorm, kblocks, S;
  int rows;  // tokens per tile (<= 128): a tile's MMA rows past it belong to the next tile
  // Shared-memory ring: `stages` slots of `stage_bytes` (x tile of `a_slot` bytes, then the
  // W_r chunks); each slot's barrier expects `tx_bytes`; barriers start at `bar_off`.
  int a_slot, stage_bytes, stages, tx_bytes, bar_off;
  int vec_logits;  // logits_out is 16-byte aligned: the split form stores rows as float4
  unsigned* status;
  unsigned long long limit_ns;
};

constexpr int R_MAX_STAGES = 32;
constexpr int R_SMEM_MAX = 227 * 1024;

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* status,
                                          uint64_t limit) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try(bar, parity)) {
    if (globaltimer_ns() - t0 > limit) {
      report(status, MOE_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_rank(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  return remote;
}
__device__ __forceinline__ float ld_dsmem(uint32_t remote_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote_addr) : "memory");
  return v;
}

// Top-KM list (KM = 2, 4 or 8 >= K), descending by (value, then lower id); empty slots
// have id -1. Ids arrive in ascending order, so an existing entry with an equal value stays
// above the new one (ties go to the lower id, +0 == -0). The top-K is the first K slots.
// Every index is a compile-time constant, so the list lives in registers.
template <int KM>
__device__ __forceinline__ void top_insert(float (&bv)[KM], int (&be)[KM], float v, int e) {
  if (be[KM - 1] >= 0 && !(v > bv[KM - 1])) return;  // does not enter
  bool above[KM];  // the entry in slot j stays above the new one
#pragma unroll
  for (int j = 0; j < KM; ++j) above[j] = be[j] >= 0 && !(v > bv[j]);
#pragma unroll
  for (int j = KM - 1; j >= 1; --j) {
    if (!above[j]) {
      if (above[j - 1]) {
        bv[j] = v;
        be[j] = e;
      } else {
        bv[j] = bv[j - 1];
        be[j] = be[j - 1];
      }
    }
  }
  if (!above[0]) {
    bv[0] = v;
    be[0] = e;
  }
}

// Columns c0..c0+15 of this warp's 32 TMEM lanes (zeros when the CTA accumulated nothing).
__device__ __forceinline__ void tmem_cols16(uint32_t trow, int c0, bool have, float (&lv)[16]) {
  uint32_t v[16];
  tmem_ld16(trow + (uint32_t)c0, v);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) lv[j] = have ? __uint_as_float(v[j]) : 0.f;
}
__device__ __forceinline__ uint32_t elect_one() {
  uint32_t p = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t.reg .b32 R;\n\telect.sync R|P, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}\n"
      : "=r"(p));
  return p;
}

template <int N, int KM>  // MMA N = E rounded up to 16; KM >= K, a power of two <= 8
__global__ void __launch_bounds__(R_THREADS) route_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                                                             const __grid_constant__ CUtensorMap tmW,
                                                             const RouteArgs g) {
  constexpr int NCH = (N + 63) / 64;         // B chunks of 64 experts
  constexpr uint32_t TCOLS = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));
  constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                             ((uint32_t)(N >> 3) << 17) | ((uint32_t)(RBM >> 4) << 24);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = base;
  const int RSTAGES = g.stages, STAGE = g.stage_bytes, A_SLOT = g.a_slot;
  uint64_t* bars = (uint64_t*)(base + g.bar_off);
  uint64_t* full = bars;
  uint64_t* empty = bars + RSTAGES;
  uint64_t* accf = bars + 2 * RSTAGES;
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * RSTAGES + 1);
  float* part = (float*)ring;  // after the mainloop: this CTA's partial, [N][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int tile = (int)cluster_id_x();
  const int S = g.S;
  const int kb0 = (int)(rank * g.kblocks / S), kb1 = (int)((rank + 1) * g.kblocks / S);
  // Tiles start their k-blocks at different points of the range (and wrap), so that the
  // CTAs do not all read the same W_r rows from the same L2 lines at the same time.
  const int nkb = kb1 - kb0, rot = nkb > 0 ? tile % nkb : 0;

  if (tid == 32) {  // fetch both tensor maps while the barriers are set up
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < RSTAGES; ++s) {
      mbar_init(saddr(&full[s]), 1);
      mbar_init(saddr(&empty[s]), 1);
    }
    mbar_init(saddr(accf), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(tmem_slot)),
                 "r"(TCOLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();

  // Producer (warp 0) and MMA issuer (warp 1) run their loops warp-uniformly: lane 0 waits
  // on the barrier and broadcasts the outcome, one elected lane issues. A single-lane loop
  // issued about a third fewer small-N MMAs per cycle (the loop, not the tensor pipe, limits
  // the rate at N = 16).
  if (warp == 0) {
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      const int kb = kb0 + (i + rot) % nkb;
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&empty[stage]), phase ^ 1u, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) {
        ok = false;
        break;
      }
      if (elect_one()) {
        const uint32_t fb = saddr(&full[stage]);
        mbar_expect_tx(fb, (uint32_t)g.tx_bytes);
        const uint32_t a = saddr(ring + stage * STAGE);
        tma_load_2d(a, &tmX, kb * RBK, tile * g.rows, fb);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          tma_load_2d(a + A_SLOT + c * RB_CHUNK, &tmW, c * 64, kb * RBK, fb);
      }
      __syncwarp();
      if (++stage == RSTAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1) {
    // Descriptors of stage 0; a stage (and a 16-wide k step) moves the start-address field,
    // which holds shared-memory byte addresses / 16 (below 2^14, so adding does not carry).
    const uint64_t ad0 = desc_sw128(saddr(ring), 16, 1024);
    const uint64_t bd0 = desc_sw128(saddr(ring) + A_SLOT, RB_CHUNK, 1024);
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&full[stage]), phase, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) {
        ok = false;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (elect_one()) {
        const uint64_t so = (uint64_t)((stage * STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < RBK / 16; ++kk) {
          const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
              "l"(ad0 + so + (uint64_t)(kk * 2)), "l"(bd0 + so + (uint64_t)(kk * 128)),
              "r"(IDESC), "r"(acc)
              : "memory");
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                saddr(&empty[stage]))
            : "memory");
      }
      __syncwarp();
      if (++stage == RSTAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (elect_one())
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              saddr(accf))
          : "memory");
  }
  __syncwarp();
  // every thread: the accumulator of this CTA is complete (bounded)
  int w_ok = 0;
  if (lane == 0) w_ok = mbar_wait(saddr(accf), 0, g.status, g.limit_ns);
  w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const bool have = w_ok && (kb1 > kb0);
  const int r = warp * 32 + lane;  // token row of this thread inside the tile
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);

  if (S > 1) {
    // Every rank publishes its partial (column-major), then after one cluster barrier each
    // rank finishes a contiguous share of the tile's rows, one thread per row, adding the S
    // partials in rank order through distributed shared memory (the same fp32 sum in the
    // same order whichever rank does it). A rank arrives on the closing barrier as soon as
    // its remote reads are done and waits on it only before exiting.
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 16) {
      float lv[16];
      tmem_cols16(trow, c0, have, lv);
#pragma unroll
      for (int j = 0; j < 16; ++j) part[(c0 + j) * RBM + r] = lv[j];
    }
    cluster_sync();
    const int share = (g.rows + S - 1) / S;
    const int row = (int)rank * share + tid;
    const bool mine = tid < share && row < g.rows;
    const int t = tile * g.rows + row;
    const int E = g.E, K = g.K;
    float bv[KM];
    int be[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      bv[k] = -INFINITY;
      be[k] = -1;
    }
    float m = -INFINITY, ssum = 0.f;  // online max / sum of exp for the plain softmax
    if (mine && t < g.T) {
      const uint32_t own = saddr(&part[row]);
#pragma unroll 1
      for (int c0 = 0; c0 < N && c0 < E; c0 += 16) {
        float lv[16];
        for (int q0 = 0; q0 < S; q0 += 4) {  // up to four ranks' loads in flight
          float pv[4][16];
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            if (q0 + qq < S) {
              const uint32_t rb = map_rank(own + (uint32_t)(c0 * RBM * 4), (uint32_t)(q0 + qq));
#pragma unroll
              for (int j = 0; j < 16; ++j) pv[qq][j] = ld_dsmem(rb + (uint32_t)(j * RBM * 4));
            }
          }
#pragma unroll
          for (int qq = 0; qq < 4; ++qq)
            if (q0 + qq < S)
#pragma unroll
              for (int j = 0; j < 16; ++j) lv[j] = q0 + qq == 0 ? pv[0][j] : lv[j] + pv[qq][j];
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int e = c0 + j;
          if (e < E) {
            if (g.bias != nullptr) lv[j] += g.bias[e];
            top_insert<KM>(bv, be, lv[j], e);
            if (!g.renorm) {
              if (lv[j] > m) {
                ssum = ssum * expf(m - lv[j]) + 1.f;
                m = lv[j];
              } else {
                ssum += expf(lv[j] - m);
              }
            }
          }
        }
        if (g.logits_out != nullptr) {  // E is a multiple of 8: whole groups of four
          float* dst = g.logits_out + (size_t)t * E + c0;
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            if (c0 + 4 * j4 < E) {
              if (g.vec_logits)
                *reinterpret_cast<float4*>(dst + 4 * j4) =
                    make_float4(lv[4 * j4], lv[4 * j4 + 1], lv[4 * j4 + 2], lv[4 * j4 + 3]);
              else
#pragma unroll
                for (int u = 0; u < 4; ++u) dst[4 * j4 + u] = lv[4 * j4 + u];
            }
          }
        }
      }
    }
    cluster_arrive();  // this rank's reads of its peers' partials are done
    if (mine && t < g.T) {
      const float top = bv[0];
      float den = 0.f;
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (k < K) den += expf(bv[k] - top);
      if (!g.renorm) den = ssum * expf(m - top);
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        if (k < K) {
          g.topk_ids[(size_t)t * K + k] = be[k];
          g.topk_w[(size_t)t * K + k] = expf(bv[k] - top) / den;
        }
      }
    }
    cluster_wait();  // no CTA exits while a peer may still read its partials
  } else {
    const int t = tile * g.rows + r;
    const int E = g.E, K = g.K;
    // Outputs are staged in this CTA's (idle) ring and written back coalesced: the tile's
    // logits rows are one contiguous [128, E] block, its ids and weights [128, K] blocks.
    float* st_l = (float*)ring;                         // [128][E + 1]
    int32_t* st_i = (int32_t*)(st_l + RBM * (E + 1));   // [128][K]
    float* st_w = (float*)(st_i + RBM * K);             // [128][K]
    float bv[KM];
    int be[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      bv[k] = -INFINITY;
      be[k] = -1;
    }
    float m = -INFINITY, ssum = 0.f;  // online max / sum of exp for the plain softmax
    const bool live = warp * 32 < g.rows;  // warp-uniform: this warp holds rows of the tile
#pragma unroll 1
    for (int c0 = 0; live && c0 < N; c0 += 16) {
      float lv[16];
      tmem_cols16(trow, c0, have, lv);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int e = c0 + j;
        float l = lv[j];
        if (e < E) {
          if (g.bias != nullptr) l += g.bias[e];
          if (t < g.T) {
            st_l[r * (E + 1) + e] = l;
            top_insert<KM>(bv, be, l, e);
            if (!g.renorm) {
              if (l > m) {
                ssum = ssum * expf(m - l) + 1.f;
                m = l;
              } else {
                ssum += expf(l - m);
              }
            }
          }
        }
      }
    }
    if (live && t < g.T) {
      const float top = bv[0];
      float den = 0.f;
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (k < K) den += expf(bv[k] - top);
      if (!g.renorm) den = ssum * expf(m - top);
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        if (k < K) {
          st_i[r * K + k] = be[k];
          st_w[r * K + k] = expf(bv[k] - top) / den;
        }
      }
    }
    __syncthreads();
    const int rows = min(g.rows, g.T - tile * g.rows);
    const size_t t0 = (size_t)tile * g.rows;
    if (g.logits_out != nullptr)
      for (int i = tid; i < rows * E; i += R_THREADS)
        g.logits_out[t0 * E + i] = st_l[(i / E) * (E + 1) + i % E];
    for (int i = tid; i < rows * K; i += R_THREADS) {
      g.topk_ids[t0 * K + i] = st_i[i];
      g.topk_w[t0 * K + i] = st_w[i];
    }
  }
  (void)ok;
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS)
                 : "memory");
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box0,
                 uint32_t box1) {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = (EncodeTiledFn)p;
  }
  cuuint64_t gd[2] = {inner, outer}, gs[1] = {inner * 2};
  cuuint32_t bx[2] = {box0, box1}, es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of S CTAs of this kernel that can be resident at once (clusters stay inside one
// GPC, so this can be below SMs / S); cached per instantiation and S.
template <typename Kern>
int active_clusters(Kern kern, int smem, int S) {
  static int cache[9] = {0};
  if (S < 1 || S > 8) return 1;
  if (cache[S] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S);
    cfg.blockDim = dim3(R_THREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = (unsigned)S;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 1;
    }
    cache[S] = n;
  }
  return cache[S];
}

// Shared-memory ring for N-wide W_r chunks. own: one tile of `rows` tokens per CTA, x slots
// of ceil(rows/8) KB and as many stages as fit (the last slot's 128-row MMA read may run
// 16 KB past its start, so the ring is padded to cover it); otherwise 128-row x slots at
// route_stages(N) deep. Returns the dynamic shared memory size, or 0 if the epilogue's
// staging buffers would not fit in the ring.
int ring_layout(int N, int E, int K, bool own, int rows, RouteArgs& a) {
  const int nch = (N + 63) / 64;
  a.a_slot = own ? ((rows + 7) / 8) * 1024 : RA_BYTES;
  a.stage_bytes = a.a_slot + nch * RB_CHUNK;
  a.tx_bytes = own ? rows * 128 + nch * RB_CHUNK : a.stage_bytes;
  auto ring_of = [&](int st) { return max(st * a.stage_bytes, (st - 1) * a.stage_bytes + RA_BYTES); };
  auto smem_of = [&](int st) { return 1024 + ring_of(st) + (2 * st + 2) * 8; };
  int st = own ? R_MAX_STAGES : route_stages(N);
  if (own)
    while (st > 2 && smem_of(st) > R_SMEM_MAX) --st;
  a.stages = st;
  a.bar_off = ring_of(st);
  const int staging = RBM * (E + 1) * 4 + 2 * RBM * K * 4;
  const int partials = N * RBM * 4;
  if (smem_of(st) > R_SMEM_MAX || ring_of(st) < staging || ring_of(st) < partials) return 0;
  return smem_of(st);
}

template <int N, int KM>
moe_status launch_nk(const void* x, const void* w_r, RouteArgs a, int tiles, bool own,
                     cudaStream_t st) {
  auto kern = route_tc_kernel<N, KM>;
  int smem = own ? ring_layout(N, a.E, a.K, true, a.rows, a) : 0;
  if (smem == 0 && own) {  // the ring does not fit: one 128-token tile per CTA, no split
    own = false;
    a.rows = RBM;
    a.S = 1;
    tiles = (a.T + RBM - 1) / RBM;
  }
  if (smem == 0) {  // one tile of up to 128 tokens per cluster of S CTAs
    smem = ring_layout(N, a.E, a.K, false, RBM, a);
    if (smem == 0) return MOE_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  // With fewer 128-token tiles than clusters that fit at once, shorter tiles (at least 64
  // tokens) put more SMs to work; the MMA still computes 128 rows, the surplus unwritten.
  if (!own && a.S > 1) {
    const int fit = active_clusters(kern, smem, a.S);
    const int want = min(fit, (a.T + 63) / 64);
    if (want > tiles) {
      a.rows = (a.T + want - 1) / want;
      tiles = (a.T + a.rows - 1) / a.rows;
    }
  }
  CUtensorMap mx, mw;
  if (!make_map_2d(&mx, x, (uint64_t)(a.kblocks * RBK), (uint64_t)a.T, 64, own ? a.rows : RBM))
    return MOE_ERR_CUDA;
  if (!make_map_2d(&mw, w_r, (uint64_t)a.E, (uint64_t)(a.kblocks * RBK), 64, 64)) return MOE_ERR_CUDA;
  launch_begin(K_ROUTE_TC, st);
  launch_kernel(kern, dim3((unsigned)(tiles * a.S)), dim3(R_THREADS), (size_t)smem, st,
                (unsigned)a.S, mx, mw, a);
  return launch_end(K_ROUTE_TC, st);
}

template <int KM>
moe_status launch_n(int N, const void* x, const void* w_r, const RouteArgs& a, int tiles,
                    bool own, cudaStream_t st) {
  if (N <= 16) return launch_nk<16, KM>(x, w_r, a, tiles, own, st);
  if (N <= 32) return launch_nk<32, KM>(x, w_r, a, tiles, own, st);
  if (N <= 64) return launch_nk<64, KM>(x, w_r, a, tiles, own, st);
  if (N <= 128) return launch_nk<128, KM>(x, w_r, a, tiles, own, st);
  return launch_nk<256, KM>(x, w_r, a, tiles, own, st);
}

}  // namespace

int g_route_layout = 0;

bool route_tc_supported(const moe_shape& s) {
  return s.dtype == MOE_BF16 && s.E % 8 == 0 && s.E <= 256 && s.K <= KMAX && s.d % 64 == 0;
}

moe_status launch_route_tc(const moe_shape& s, const void* x, const void* w_r, const float* bias,
                           float* logits_out, int32_t* ids, float* w, cudaStream_t st) {
  int tiles = (s.T + RBM - 1) / RBM;
  const int kblocks = s.d / RBK;
  const int N = ((s.E + 15) / 16) * 16;  // MMA N (a multiple of 16 for M = 128)
  const int nmma = N <= 16 ? 16 : N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  // On request, one tile of ceil(T / SMs) <= 128 tokens per CTA over the whole of d (no
  // split, no cluster). Not the default: it issues one M = 128 MMA per 16-wide k step for
  // fewer useful rows, and the MMA issue loop, not HBM, bounds this kernel.
  const int rows_own = (s.T + sm_count() - 1) / sm_count();
  const bool own = g_route_layout == 2 && rows_own <= RBM;
  int S = 1;
  if (!own) {
    // Split d over S CTAs so that about one CTA per SM works, but never beyond the CTAs
    // that can be resident at once (a second wave costs more than the split saves).
    const int smem_cta =
        route_stages(nmma) * (RA_BYTES + ((nmma + 63) / 64) * RB_CHUNK) + 1024 + 256;
    const int per_sm = R_SMEM_MAX / smem_cta;
    S = (sm_count() + tiles - 1) / tiles;
    const int resident = sm_count() * (per_sm > 0 ? per_sm : 1);
    if (S > resident / tiles) S = resident / tiles;
    if (S > 8) S = 8;
    if (S > kblocks) S = kblocks;
    if (S < 1) S = 1;
  }
  RouteArgs a;
  a.bias = bias;
  a.logits_out = logits_out;
  a.topk_ids = ids;
  a.topk_w = w;
  a.T = s.T;
  a.E = s.E;
  a.K = s.K;
  a.renorm = s.renormalize;
  a.kblocks = kblocks;
  a.S = S;
  a.rows = own ? rows_own : RBM;
  a.vec_logits = ((uintptr_t)logits_out & 15) == 0;
  if (own) tiles = (s.T + a.rows - 1) / a.rows;
  a.status = device_status_ptr();
  a.limit_ns = kWaitLimitNs;
  // instantiations cover N up to the next of 16/32/64/128/256; columns past E read zeros
  if (s.K <= 2) return launch_n<2>(N, x, w_r, a, tiles, own, st);
  if (s.K <= 4) return launch_n<4>(N, x, w_r, a, tiles, own, st);
  return launch_n<8>(N, x, w_r, a, tiles, own, st);
}

}  // namespace moe
