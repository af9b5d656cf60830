// bf16 grouped SwiGLU FFN on CTA pairs: tcgen05.mma.cta_group::2, 256 x 256 tiles.
//
// Same method as the single-CTA kernel (SonicMoE explainer, gitcode.csdn.net, section 3
// items 3-5; section 6.2 gather fusion; section 6.3 epilogue fusion), with the tile spread
// over a cluster of two CTAs on two SMs. The pair computes 256 rows x 256 columns: each
// CTA holds its own 128 rows of A and half (128 columns) of B in its shared memory, and
// the MMA issued by the pair's leader (rank 0) reads both CTAs' halves, writing each CTA's
// 128 x 256 fp32 accumulator into that CTA's TMEM. Per SM and per k-block this moves
// 32 KB (16 KB of A + 16 KB of B) instead of the single-CTA kernel's 48 KB, so six stages
// fit in shared memory and cover more memory latency.
//   gate/up: rank 0 holds the W_gate columns n0..n0+127, rank 1 the W_up columns, so every
//   thread still finds its row's (gate, up) pairs in TMEM columns c and 128 + c.
//   down:    rank r holds W_down columns n0 + 128 r .. + 127.
//   backward dX (MODE 3): dX_perm = (dG | dU) (W_gate | W_up)^T: A = the d_h rows by TMA,
//   B K-major (rank r holds rows n0 + 128 r .. + 127 of W_gate[e], or of W_up[e] for the
//   second half of the contraction, read in place as the transposes).
// Synchronisation: TMA loads of both CTAs (.cta_group::2) complete on the leader's full
// barrier; gate/up gathers by cp.async complete on the leader's barrier directly (leader)
// or on a local barrier that one peer thread relays to the leader after a proxy fence
// (peer); the leader commits each stage to both CTAs' empty barriers and each tile to both
// CTAs' accumulator-full barriers; both CTAs' epilogue warps arrive on the leader's
// accumulator-empty barrier. Every wait is bounded (MOE_ERR_TIMEOUT on expiry).
#include "ffn_args.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace {

using namespace ptx;

constexpr int BM = 128;  // rows per CTA; the pair covers PAIR_M
constexpr int PAIR_M = 256;
constexpr int BK = 64, BN = 256, STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_CHUNK = BK * 64 * 2;          // 8 KB: 64 k-rows x 64 columns
constexpr int B_HALF = 2 * B_CHUNK;           // this CTA's 128 of the 256 MMA columns
constexpr int STAGE_BYTES = A_BYTES + B_HALF; // 32 KB
constexpr int THREADS_DOWN = 192;
constexpr int THREADS_GATEUP = 320;
constexpr int GATHER_WARP0 = 6;
constexpr int GATHER_THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAXE = 256;
constexpr int SMEM_TAIL = 4096;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + SMEM_TAIL;
constexpr uint32_t IDESC = idesc_bf16(PAIR_M, BN);
constexpr uint32_t IDESC_BK = IDESC & ~(1u << 16);  // B K-major (backward dX)


struct Tile2 {
  int e, m0, rows, n0, m0_pair;  // m0 / rows: this CTA's half of the pair's 256 rows
};

__device__ __forceinline__ Tile2 decode2(int w, const int* s_off, const int* s_cum,
                                         const int* s_mt, int E, int out_tile, uint32_t rank) {
  int lo = 0, hi = E - 1;  // largest e with s_cum[e] <= w
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_cum[mid] <= w) lo = mid;
    else hi = mid - 1;
  }
  Tile2 t;
  t.e = lo;
  const int local = w - s_cum[lo];
  const int mt = s_mt[lo];
  t.n0 = (local / mt) * out_tile;
  t.m0_pair = s_off[lo] + (local % mt) * PAIR_M;
  t.m0 = t.m0_pair + (int)rank * BM;
  t.rows = max(0, min(BM, s_off[lo + 1] - t.m0));
  return t;
}

// MODE 0: down GEMM (A = the activations, by TMA); 1: gate/up GEMM with the A rows
// gathered from x by cp.async; 2: gate/up GEMM with A = rows already gathered into an
// expert-major buffer, by TMA (no gather warps, no relay); 3: backward dX (A = the d_h
// rows by TMA, B K-major from W_gate then W_up).
template <int MODE>
__global__ void __launch_bounds__(MODE == 1 ? THREADS_GATEUP : THREADS_DOWN, 1)
    grouped_gemm_tc2(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB0,
                     const __grid_constant__ CUtensorMap tmB1, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = base;
  uint64_t* bars = (uint64_t*)(base + STAGES * STAGE_BYTES);
  uint64_t* full = bars;                   // leader: the stage's A and B landed in both CTAs
  uint64_t* empty = bars + STAGES;         // both: the MMAs reading the stage completed
  uint64_t* gfull = bars + 2 * STAGES;     // peer: its gathered A rows landed (gate/up)
  uint64_t* tfull = bars + 3 * STAGES;     // both: accumulator b complete
  uint64_t* tempty = bars + 3 * STAGES + 2;  // leader: both CTAs drained accumulator b
  uint64_t* done = bars + 3 * STAGES + 4;
  uint32_t* tmem_slot = (uint32_t*)(bars + 3 * STAGES + 5);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  int* s_off = (int*)(tmem_slot + 2);
  int* s_cum = s_off + MAXE + 1;
  int* s_mt = s_cum + MAXE + 1;

  constexpr bool GATEUP = MODE == 1 || MODE == 2;
  constexpr bool BKMAJOR = MODE == 3;
  constexpr bool GATHER = MODE == 1;
  constexpr int NTHREADS = GATHER ? THREADS_GATEUP : THREADS_DOWN;
  // leader's full[s]: the leader's expect_tx arrival for the TMA bytes of both CTAs (+ the
  // leader's gather threads + the peer's relay). The peer's loads complete on it without
  // an arrival of their own: a transaction count may run ahead of its expect_tx, and the
  // phase cannot complete before the leader's arrival anyway.
  constexpr uint32_t FULL_COUNT = GATHER ? 1 + GATHER_THREADS + 1 : 1;
  constexpr uint32_t TMA_BYTES = GATHER ? B_HALF : STAGE_BYTES;  // per CTA and stage

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = (int)cluster_id_x(), npairs = (int)num_clusters_x();
  const int E = g.E;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(saddr(&full[s]), FULL_COUNT);
      mbar_init(saddr(&empty[s]), 1);
      mbar_init(saddr(&gfull[s]), GATHER_THREADS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(saddr(&tfull[b]), 1);
      mbar_init(saddr(&tempty[b]), 8);  // 4 epilogue warps x 2 CTAs
    }
    mbar_init(saddr(done), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc<2>(saddr(tmem_slot), TMEM_COLS);
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  for (int i = tid; i <= E; i += NTHREADS) s_off[i] = g.offsets[i];
  __syncthreads();
  if (warp == 0) {  // tile table: s_mt[e] = ceil(kept_e / 256); s_cum = n_tiles * prefix
    constexpr int PER = MAXE / 32;
    int loc[PER], sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane * PER + j;
      loc[j] = (e < E) ? (s_off[e + 1] - s_off[e] + PAIR_M - 1) / PAIR_M : 0;
      sum += loc[j];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane * PER + j;
      if (e < E) {
        s_mt[e] = loc[j];
        s_cum[e] = run * g.n_tiles;
      }
      run += loc[j];
    }
    if (lane == 31) s_cum[E] = incl * g.n_tiles;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_cum[E];
  const uint64_t limit = g.limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_par = 0;  // per stage: ever issued, parity of last issue
    for (int w = pair; w < total; w += npairs) {
      const Tile2 t = decode2(w, s_off, s_cum, s_mt, E, g.out_tile, rank);
      bool ok = true;
      for (int kb = 0; kb < g.kblocks; ++kb) {
        int w_ok = 0;
        if (lane == 0)
          w_ok = mbar_wait<true>(saddr(&empty[stage]), phase ^ 1u, abort_flag, g.status, limit);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        const uint32_t fb = map_rank(saddr(&full[stage]), 0);  // the leader's barrier
        if (leader && lane == 0) mbar_expect_tx(saddr(&full[stage]), 2 * TMA_BYTES);
        __syncwarp();
        const uint32_t a_dst = saddr(ring + stage * STAGE_BYTES);
        const uint32_t b_dst = a_dst + A_BYTES;
        if (!GATHER && lane == 0) tma_load_2d_pair(a_dst, &tmA, kb * BK, t.m0, fb);
        if (BKMAJOR) {
          if (lane == 0) {
            const bool first = kb < g.kb_split;
            tma_load_3d_pair(b_dst, first ? &tmB0 : &tmB1, (first ? kb : kb - g.kb_split) * BK,
                             t.n0 + (int)rank * 128, t.e, fb);
          }
        } else if (lane < 2) {
          if (GATEUP)
            tma_load_3d_pair(b_dst + lane * B_CHUNK, leader ? &tmB0 : &tmB1, t.n0 + lane * 64,
                             kb * BK, t.e, fb);
          else
            tma_load_3d_pair(b_dst + lane * B_CHUNK, &tmB0, t.n0 + (int)rank * 128 + lane * 64,
                             kb * BK, t.e, fb);
        }
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    // The leader's full barriers count both CTAs' bytes: once the last phase issued into
    // each stage completed (bounded), no load of the pair is in flight. The peer waits for
    // this at the final cluster barrier.
    if (leader && lane == 0) {
      for (int s = 0; s < STAGES; ++s) {
        if (!(issued_mask & (1u << s))) continue;
        const uint32_t par = (issued_par >> s) & 1u;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_cluster(saddr(&full[s]), par) && globaltimer_ns() - t0 < limit) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ---------------------------------------------------------- MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int w = pair; w < total && ok; w += npairs, ++it) {
        const int buf = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait<true>(saddr(&tempty[buf]), (use & 1u) ^ 1u, abort_flag, g.status, limit))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait<true>(saddr(&full[stage]), phase, abort_flag, g.status, limit)) {
            ok = false;
            break;
          }
          if (GATHER) fence_proxy_async_smem();  // this CTA's cp.async rows -> MMA reads
          tc_fence_after();
          const uint32_t a_addr = saddr(ring + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = BKMAJOR ? desc_sw128(b_addr + kk * 32, 16, 1024)
                                        : desc_sw128(b_addr + kk * 2048, B_CHUNK, 1024);
            tc_mma<2>(d_tmem, ad, bd, BKMAJOR ? IDESC_BK : IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit<2>(saddr(&empty[stage]));
          tc_commit<2>(map_rank(saddr(&empty[stage]), 1));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) {
          tc_commit<2>(saddr(&tfull[buf]));
          tc_commit<2>(map_rank(saddr(&tfull[buf]), 1));
        }
      }
      tc_commit<2>(saddr(done));  // every MMA of the pair completed before TMEM is freed
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try(saddr(done), 0) && globaltimer_ns() - t0 < limit) {
      }
    } else if (GATHER && !leader && lane == 0) {
      // ---------------------------------------------------------- gather relay (peer)
      int stage = 0;
      uint32_t phase = 0;
      for (int w = pair; w < total; w += npairs) {
        bool ok = true;
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait<false>(saddr(&gfull[stage]), phase, abort_flag, g.status, limit)) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();  // this CTA's cp.async rows -> the leader's MMA reads
          mbar_arrive_remote(map_rank(saddr(&full[stage]), 0));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else if (GATHER && warp >= GATHER_WARP0) {
    // ------------------------------------------------------------ A gather (both CTAs)
    const int gw = warp - GATHER_WARP0;
    const int c = lane & 7;
    const int rg = lane >> 3;
    auto rows_of = [&](int w, const uint8_t* (&src)[8]) {
      const Tile2 t = decode2(w, s_off, s_cum, s_mt, E, g.out_tile, rank);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = gw * 32 + rg + 4 * i;
        // padding rows (and a half with no rows) reuse the pair's first row
        const int p = r < t.rows ? t.m0 + r : t.m0_pair;
        const int a = g.p2a[p];
        int tk = a / g.K;
        if (a < 0 || tk >= g.T) {
          report(g.status, MOE_ERR_DEVICE_INDEX);
          tk = 0;
        }
        src[i] = g.x + (size_t)tk * g.x_row_bytes + c * 16;
      }
    };
    uint32_t dst[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = gw * 32 + rg + 4 * i;
      dst[i] = (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));  // 128-byte swizzle
    }
    uint64_t* land = leader ? full : gfull;
    int stage = 0;
    uint32_t phase = 0;
    const uint8_t* src[8];
    if (pair < total) rows_of(pair, src);
    for (int w = pair; w < total; w += npairs) {
      const uint8_t* nsrc[8];
      if (w + npairs < total) rows_of(w + npairs, nsrc);
      bool ok = true;
      for (int kb = 0; kb < g.kblocks; ++kb) {
        int w_ok = 0;
        if (lane == 0)
          w_ok = mbar_wait<true>(saddr(&empty[stage]), phase ^ 1u, abort_flag, g.status, limit);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        const uint32_t a_dst = saddr(ring + stage * STAGE_BYTES);
#pragma unroll
        for (int i = 0; i < 8; ++i) cp_async16(a_dst + dst[i], src[i] + (size_t)kb * (BK * 2));
        cp_async_arrive_noinc(saddr(&land[stage]));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
#pragma unroll
      for (int i = 0; i < 8; ++i) src[i] = nsrc[i];
    }
    cp_async_wait_all();
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t tempty_leader = map_rank(saddr(&tempty[0]), 0);
    int it = 0;
    for (int w = pair; w < total; w += npairs, ++it) {
      const Tile2 t = decode2(w, s_off, s_cum, s_mt, E, g.out_tile, rank);
      const int buf = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      int w_ok = 0;
      if (lane == 0)
        w_ok = mbar_wait<true>(saddr(&tfull[buf]), use & 1u, abort_flag, g.status, limit);
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (!w_ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (uint32_t)(buf * BN) + ((uint32_t)(q * 32) << 16);
      const bool row_ok = r < t.rows;
      bf16* orow = g.out + (size_t)(t.m0 + (row_ok ? r : 0)) * g.ld_out;
      if (GATEUP) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tb + c * 32, gv);
          tmem_ld32(tb + 128 + c * 32, uv);
          tmem_ld_wait();
          const int col = t.n0 + c * 32;
          if (row_ok && col < g.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g0 = __uint_as_float(gv[2 * j]), g1 = __uint_as_float(gv[2 * j + 1]);
              const float u0 = __uint_as_float(uv[2 * j]), u1 = __uint_as_float(uv[2 * j + 1]);
              pk[j] = pack_bf16x2(__fdividef(g0, 1.f + __expf(-g0)) * u0, __fdividef(g1, 1.f + __expf(-g1)) * u1);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tb + c * 32, v);
          tmem_ld_wait();
          const int col = t.n0 + c * 32;
          if (row_ok && col < g.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader + (uint32_t)(buf * 8));
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair is done with both TMEM allocations and all barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<2>(tmem_base, TMEM_COLS);
  }
}

template <int MODE>
moe_status run_gemm2(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                     const GemmArgs& args, cudaStream_t st, int kid) {
  auto kern = grouped_gemm_tc2<MODE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  const int pairs = sm_count() / 2;
  launch_begin(kid, st);
  launch_kernel(kern, dim3((unsigned)(2 * (pairs > 0 ? pairs : 1))),
                dim3(MODE == 1 ? THREADS_GATEUP : THREADS_DOWN), (size_t)SMEM_BYTES, st, 2, a, b0,
                b1, args);
  return launch_end(kid, st);
}

}  // namespace

moe_status launch_ffn_tc2_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0,
                               const CUtensorMap& b1, const GemmArgs& args, cudaStream_t st) {
  if (mode == 1) return run_gemm2<1>(a, b0, b1, args, st, K_GATEUP_TC2);
  if (mode == 2) return run_gemm2<2>(a, b0, b1, args, st, K_GATEUP_TC2);
  if (mode == 3) return run_gemm2<3>(a, b0, b1, args, st, K_BWD_DX);
  return run_gemm2<0>(a, b0, b1, args, st, K_DOWN_TC2);
}

}  // namespace moe
