// Dispatch metadata: per-expert counts, capacity clamp, exclusive scan and the stable
// permutation between token-major assignments and expert-major slots.
//
// "Operators & compilers: MoE routing and sparse kernels" (charles2530.github.io),
// section 3: regrouping tokens by expert is an index/scatter/gather problem that needs
// counting and a prefix sum; section 4: a capacity factor bounds each expert's tokens and
// the overflow is dropped. "Two upstream innovations of MoE: Routing-Free and OmniMoE"
// (chatdocs.ruinique.com), section 2.3: tasks sorted by (expert, token). SonicMoE explainer
// (gitcode.csdn.net), section 11: counts per expert, slot -> token, token slot -> slot.
//
// Atomic-free and deterministic. The T*K flat assignments are cut into chunks of
// kChunk (1024); a CTA owns a chunk and each of its 8 warps a contiguous slice of it.
//   hist    : per warp, 32 ids at a time, __match_any_sync groups equal ids and the
//             group's lowest lane adds the group size to the warp's private counter row
//             (no two lanes touch one address); the CTA sums its 8 rows per expert.
//   scan    : one CTA of 1024 threads, several per expert: each sums a run of chunks, a
//             segmented prefix over the runs gives every chunk's rank base inside its
//             expert; counts[e] is the total, kept = min(count, C) and offsets = exclusive
//             scan of kept over experts. When chunks x experts is small the scatter CTAs
//             derive their own bases and the offsets instead (two launches, not three).
//   scatter : recomputes the warp rows, turns them into rank bases (chunk base + earlier
//             warps), then walks the slice again: rank = base + (lanes of the group below
//             me); rank < C -> slot offsets[e] + rank, else dropped (-1).
// Problems of at most kSmallMax assignments run all three phases in one CTA.
// Inside an expert the slots follow ascending flat index a = t*K + k, i.e. token order.
#include <algorithm>
#include <mutex>
#include <type_traits>

#include "tc_ptx.cuh"
#include "topk.cuh"
#include "round.cuh"

namespace moe {

namespace {

constexpr int kWarps = 8;
constexpr int kIters = 4;                    // 32-id groups per warp
constexpr int kSlice = 32 * kIters;          // ids per warp
constexpr int kChunk = kWarps * kSlice;      // ids per CTA
constexpr int kMaxE = 256;

// Ids are fetched with plain non-coherent loads first and validated afterwards, so that a
// group of loads is issued back to back (a status report between loads would serialise
// them). An id outside [0, E) is reported and treated as absent.
__device__ __forceinline__ int raw_id(const int32_t* __restrict__ ids, long long a, long long A) {
  return a < A ? __ldg(ids + a) : -1;
}
__device__ __forceinline__ int checked_id(int id, bool real, int E, unsigned* status) {
  if (!real || id == -1) return -1;  // -1: no expert (an assignment removed by rounding)
  if (id < 0 || id >= E) {
    report(status, MOE_ERR_DEVICE_INDEX);
    return -1;
  }
  return id;
}

// Counts of this warp's slice into its private row (plain shared-memory adds by unique lanes).
__device__ __forceinline__ void warp_histogram(const int32_t* ids, long long slice0, long long A,
                                               int E, int* row, unsigned* status) {
  const int lane = threadIdx.x & 31;
  int v[kIters];
#pragma unroll
  for (int it = 0; it < kIters; ++it) v[it] = raw_id(ids, slice0 + it * 32 + lane, A);
#pragma unroll
  for (int it = 0; it < kIters; ++it) v[it] = checked_id(v[it], slice0 + it * 32 + lane < A, E, status);
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const unsigned m = __match_any_sync(0xffffffffu, v[it]);
    if (v[it] >= 0 && lane == __ffs(m) - 1) row[v[it]] += __popc(m);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kWarps * 32) hist_kernel(const int32_t* __restrict__ ids,
                                                           long long A, int E,
                                                           int32_t* __restrict__ chunk_counts,
                                                           unsigned* status) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  __shared__ int rows[kWarps][kMaxE];
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < kWarps * kMaxE; i += blockDim.x) (&rows[0][0])[i] = 0;
  __syncthreads();
  const long long slice0 = (long long)blockIdx.x * kChunk + (long long)warp * kSlice;
  warp_histogram(ids, slice0, A, E, rows[warp], status);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += rows[w][e];
    chunk_counts[(size_t)blockIdx.x * E + e] = s;
  }
}

// Chunk rank bases for many chunks: one CTA of kScanThreads threads, kScanThreads / Epad
// of them per expert (Epad = E rounded up to a power of two), each owning a run of
// consecutive chunks.
constexpr int kScanThreads = 1024;
constexpr long long kFusedScanMax = 8192;  // chunks x experts summed by every scatter CTA

__global__ void __launch_bounds__(kScanThreads) scan_kernel(
    const int32_t* __restrict__ chunk_counts, int32_t* __restrict__ chunk_base, int nchunks, int E,
    int Epad, long long cap, int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  __shared__ long long part[kScanThreads];
  __shared__ long long kept_s[kMaxE];
  const int tid = threadIdx.x;
  const int tpe = kScanThreads / Epad;  // threads per expert
  const int e = tid / tpe, j = tid % tpe;
  const int seg = (nchunks + tpe - 1) / tpe;
  const int c0 = min(nchunks, j * seg), c1 = min(nchunks, c0 + seg);
  long long sum = 0;
  if (e < E) {
    int c = c0;
    for (; c + 8 <= c1; c += 8) {  // eight independent loads in flight
      int v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = chunk_counts[(size_t)(c + q) * E + e];
#pragma unroll
      for (int q = 0; q < 8; ++q) sum += v[q];
    }
    for (; c < c1; ++c) sum += chunk_counts[(size_t)c * E + e];
  }
  part[tid] = sum;
  __syncthreads();
  for (int off = 1; off < tpe; off <<= 1) {  // inclusive prefix inside each expert's group
    const long long add = (j >= off) ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += add;
    __syncthreads();
  }
  if (e < E) {
    long long run = part[tid] - sum;  // exclusive: chunks before this run
    for (int c = c0; c < c1; ++c) {
      chunk_base[(size_t)c * E + e] = (int32_t)run;
      run += chunk_counts[(size_t)c * E + e];
    }
  }
  if (j == tpe - 1 && e < kMaxE) {
    const long long total = (e < E) ? part[tid] : 0;
    if (e < E) counts[e] = (int32_t)total;
    kept_s[e] = (e < E) ? (cap >= 0 && total > cap ? cap : total) : 0;
  }
  __syncthreads();
  for (int off = 1; off < Epad; off <<= 1) {  // inclusive scan of kept over experts
    long long add = 0;
    if (tid < Epad && tid >= off) add = kept_s[tid - off];
    __syncthreads();
    if (tid < Epad) kept_s[tid] += add;
    __syncthreads();
  }
  if (tid < E) {
    const long long prev = tid > 0 ? kept_s[tid - 1] : 0;
    offsets[tid] = (int32_t)prev;
    if (tid == E - 1) offsets[E] = (int32_t)kept_s[tid];
  }
}

// fused_scan: chunk_base is not given; every CTA sums the chunk counts itself (its bases:
// chunks before it; the offsets: all chunks) and CTA 0 also writes counts and offsets.
__global__ void __launch_bounds__(kWarps * 32) scatter_kernel(
    const int32_t* __restrict__ ids, long long A, int E, long long cap,
    const int32_t* __restrict__ chunk_counts, const int32_t* __restrict__ chunk_base,
    int nchunks, int fused_scan, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ assign_to_perm, int32_t* __restrict__ perm_to_assign, unsigned* status) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  __shared__ int rows[kWarps][kMaxE];
  __shared__ int offs[kMaxE];
  __shared__ int cbase[kMaxE];
  __shared__ long long kept_s[kMaxE];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kWarps * kMaxE; i += blockDim.x) (&rows[0][0])[i] = 0;
  if (!fused_scan) {
    for (int e = tid; e < E; e += blockDim.x) {
      offs[e] = offsets[e];
      cbase[e] = chunk_base[(size_t)blockIdx.x * E + e];
    }
  } else {
    for (int e = tid; e < kMaxE; e += blockDim.x) {
      long long before = 0, total = 0;
      if (e < E) {
        for (int c = 0; c < nchunks; ++c) {
          const int v = chunk_counts[(size_t)c * E + e];
          if (c < (int)blockIdx.x) before += v;
          total += v;
        }
        if (blockIdx.x == 0) counts[e] = (int32_t)total;
      }
      cbase[e] = (int)before;
      kept_s[e] = (e < E) ? (cap >= 0 && total > cap ? cap : total) : 0;
    }
    __syncthreads();
    for (int off = 1; off < kMaxE; off <<= 1) {  // inclusive scan of kept over experts
      long long add[kMaxE / (kWarps * 32)];
#pragma unroll
      for (int q = 0; q < kMaxE / (kWarps * 32); ++q) {
        const int e = tid + q * kWarps * 32;
        add[q] = e >= off ? kept_s[e - off] : 0;
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < kMaxE / (kWarps * 32); ++q) kept_s[tid + q * kWarps * 32] += add[q];
      __syncthreads();
    }
    for (int e = tid; e < E; e += blockDim.x) {
      offs[e] = (int)(e > 0 ? kept_s[e - 1] : 0);
      if (blockIdx.x == 0) {
        offsets[e] = offs[e];
        if (e == E - 1) offsets[E] = (int32_t)kept_s[e];
      }
    }
  }
  __syncthreads();
  const long long slice0 = (long long)blockIdx.x * kChunk + (long long)warp * kSlice;
  warp_histogram(ids, slice0, A, E, rows[warp], nullptr);
  __syncthreads();
  // rank base of each warp row: chunk base + counts of the earlier warps of this chunk
  for (int e = tid; e < E; e += blockDim.x) {
    int run = cbase[e];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = rows[w][e];
      rows[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  int* base = rows[warp];
  const unsigned lt = lanemask_lt();
  int v[kIters];
#pragma unroll
  for (int it = 0; it < kIters; ++it) v[it] = raw_id(ids, slice0 + it * 32 + lane, A);
#pragma unroll
  for (int it = 0; it < kIters; ++it) v[it] = checked_id(v[it], slice0 + it * 32 + lane < A, E, nullptr);
#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const long long a = slice0 + it * 32 + lane;
    const int id = v[it];
    const unsigned m = __match_any_sync(0xffffffffu, id);
    int rank = 0;
    if (id >= 0) rank = base[id] + __popc(m & lt);
    __syncwarp();
    if (id >= 0 && lane == __ffs(m) - 1) base[id] += __popc(m);
    __syncwarp();
    if (id >= 0) {
      int p = -1;
      if (cap < 0 || rank < cap) {
        p = offs[id] + rank;
        perm_to_assign[p] = (int32_t)a;
      }
      assign_to_perm[a] = p;
    } else if (a < A) {
      assign_to_perm[a] = -1;  // id out of range (already reported)
    }
  }
}

// Small problems (T*K <= kSmallMax): histogram, scan and scatter in one CTA of 32 warps,
// one launch instead of three. Same algorithm and same result as the three kernels: each
// warp owns a contiguous slice, counts it into its private row, the rows are turned into
// rank bases in warp order, and the slice is walked again to place each assignment.
constexpr int kSmallWarps = 32;
constexpr int kSmallIters = 2;  // 32-id groups per warp
constexpr int kGroup = 2;       // of which loaded together
constexpr long long kSmallMax = (long long)kSmallWarps * 32 * kSmallIters;  // 2048

__global__ void __launch_bounds__(kSmallWarps * 32) permute_small_kernel(
    const int32_t* __restrict__ ids, long long A, int E, long long cap, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ assign_to_perm,
    int32_t* __restrict__ perm_to_assign, unsigned* status) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  __shared__ int rows[kSmallWarps][kMaxE];
  __shared__ long long kept_s[kMaxE];
  __shared__ int offs[kMaxE];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int iters = (int)((A + kSmallWarps * 32 - 1) / (kSmallWarps * 32));  // <= kSmallIters
  const long long s0 = (long long)warp * iters * 32;
  for (int i = tid; i < kSmallWarps * kMaxE; i += blockDim.x) (&rows[0][0])[i] = 0;
  __syncthreads();
  int* row = rows[warp];
  // the slice is read in groups of kGroup ids per lane, each group one round of
  // independent loads
  for (int g0 = 0; g0 < iters; g0 += kGroup) {
    int v[kGroup];
#pragma unroll
    for (int j = 0; j < kGroup; ++j)
      v[j] = g0 + j < iters ? raw_id(ids, s0 + (g0 + j) * 32 + lane, A) : -1;
#pragma unroll
    for (int j = 0; j < kGroup; ++j)
      v[j] = checked_id(v[j], g0 + j < iters && s0 + (g0 + j) * 32 + lane < A, E, status);
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      const unsigned m = __match_any_sync(0xffffffffu, v[j]);
      if (v[j] >= 0 && lane == __ffs(m) - 1) row[v[j]] += __popc(m);
      __syncwarp();
    }
  }
  __syncthreads();
  long long run = 0;
  if (tid < kMaxE) {
    const int e = tid;
    if (e < E) {
      for (int w = 0; w < kSmallWarps; ++w) {
        const int c = rows[w][e];
        rows[w][e] = (int)run;
        run += c;
      }
      counts[e] = (int32_t)run;
    }
    kept_s[e] = (e < E) ? (cap >= 0 && run > cap ? cap : run) : 0;
  }
  __syncthreads();
  for (int off = 1; off < kMaxE; off <<= 1) {  // inclusive scan of kept over experts
    long long add = 0;
    if (tid < kMaxE && tid >= off) add = kept_s[tid - off];
    __syncthreads();
    if (tid < kMaxE) kept_s[tid] += add;
    __syncthreads();
  }
  if (tid < E) {
    const long long mine = (cap >= 0 && run > cap) ? cap : run;
    offs[tid] = (int)(kept_s[tid] - mine);
    offsets[tid] = (int32_t)(kept_s[tid] - mine);
    if (tid == E - 1) offsets[E] = (int32_t)kept_s[tid];
  }
  __syncthreads();
  const unsigned lt = lanemask_lt();
  for (int g0 = 0; g0 < iters; g0 += kGroup) {
    int v[kGroup];
#pragma unroll
    for (int j = 0; j < kGroup; ++j)
      v[j] = g0 + j < iters ? raw_id(ids, s0 + (g0 + j) * 32 + lane, A) : -1;
#pragma unroll
    for (int j = 0; j < kGroup; ++j)
      v[j] = checked_id(v[j], g0 + j < iters && s0 + (g0 + j) * 32 + lane < A, E, nullptr);
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      if (g0 + j >= iters) break;  // past this warp's slice (warp-uniform)
      const long long a = s0 + (g0 + j) * 32 + lane;
      const int id = v[j];
      const unsigned m = __match_any_sync(0xffffffffu, id);
      int rank = 0;
      if (id >= 0) rank = row[id] + __popc(m & lt);
      __syncwarp();
      if (id >= 0 && lane == __ffs(m) - 1) row[id] += __popc(m);
      __syncwarp();
      if (id >= 0) {
        int p = -1;
        if (cap < 0 || rank < cap) {
          p = offs[id] + rank;
          perm_to_assign[p] = (int32_t)a;
        }
        assign_to_perm[a] = p;
      } else if (a < A) {
        assign_to_perm[a] = -1;
      }
    }
  }
}

// Medium problems (kSmallMax < T*K <= kClusterMax): histogram, scan and scatter in one
// launch of a cluster of C <= 8 CTAs of WARPS warps, CTA c owning the contiguous chunk
// [c * WARPS * 32 * ITERS, (c + 1) * WARPS * 32 * ITERS) and each warp a slice of
// ITERS x 32 ids inside it. Same algorithm and result as the three kernels; the ids stay in
// registers between the counting and the placing walk, and the chunk counts are exchanged
// through distributed shared memory instead of global memory: after one cluster barrier
// thread e of every CTA reads the C counts of expert e (its rank base = the counts of the
// earlier CTAs, the expert's total = all of them). Each CTA then arrives on a second
// cluster barrier and waits on it only before exiting, so no CTA leaves while another may
// still read its counts, and nobody stalls for it in between.
constexpr int kClusterMaxCtas = 8;
constexpr long long kClusterMax = (long long)kClusterMaxCtas * 32 * 32 * 4;  // 32 warps x 4

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int WARPS, int ITERS>
__global__ void __launch_bounds__(WARPS * 32) permute_cluster_kernel(
    const int32_t* __restrict__ ids, long long A, int E, long long cap, int C,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ assign_to_perm, int32_t* __restrict__ perm_to_assign, unsigned* status) {
  constexpr int NT = WARPS * 32;
  static_assert(NT >= kMaxE, "one thread per expert in the scan");
  __shared__ int rows[WARPS][kMaxE];
  __shared__ int ctot[kMaxE];   // this CTA's count per expert (read by every CTA)
  __shared__ int cbase[kMaxE];  // counts of the earlier CTAs
  __shared__ int offs[kMaxE];
  __shared__ int wsum[kMaxE / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = ptx::cluster_rank();
  const long long s0 = ((long long)rank * WARPS + warp) * (32LL * ITERS);
  for (int i = tid; i < WARPS * kMaxE; i += NT) (&rows[0][0])[i] = 0;
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  int v[ITERS];
#pragma unroll
  for (int it = 0; it < ITERS; ++it) v[it] = raw_id(ids, s0 + it * 32 + lane, A);
  __syncthreads();  // rows zeroed
#pragma unroll
  for (int it = 0; it < ITERS; ++it) v[it] = checked_id(v[it], s0 + it * 32 + lane < A, E, status);
  int* row = rows[warp];
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const unsigned m = __match_any_sync(0xffffffffu, v[it]);
    if (v[it] >= 0 && lane == __ffs(m) - 1) row[v[it]] += __popc(m);
    __syncwarp();
  }
  __syncthreads();
  // per-warp exclusive bases inside the CTA and the CTA's total: warp w takes experts
  // w, w + WARPS, ...; lane l holds warp l's count and a shuffle scan runs over the lanes
  for (int e = warp; e < E; e += WARPS) {
    const int c = lane < WARPS ? rows[lane][e] : 0;
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane < WARPS) rows[lane][e] = incl - c;
    if (lane == 31) ctot[e] = incl;
  }
  ptx::cluster_sync();  // every CTA's totals are complete
  int total = 0;
  if (tid < E) {
    int cv[kClusterMaxCtas];
    const uint32_t mine = ptx::saddr(&ctot[tid]);
#pragma unroll
    for (int q = 0; q < kClusterMaxCtas; ++q)
      cv[q] = q < C ? ptx::ld_dsmem_s32(ptx::map_rank(mine, (uint32_t)q)) : 0;
    int before = 0;
#pragma unroll
    for (int q = 0; q < kClusterMaxCtas; ++q) {
      if (q < (int)rank) before += cv[q];
      total += cv[q];
    }
    cbase[tid] = before;
    if (rank == 0) counts[tid] = total;
  }
  cluster_arrive();  // this CTA's remote reads are done (waited on before exit)
  // exclusive scan of kept = min(total, cap) over the experts (threads 0..255)
  int kept = 0, incl = 0;
  if (tid < kMaxE) {
    kept = (tid < E) ? (int)((cap >= 0 && total > cap) ? cap : total) : 0;
    incl = kept;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
  }
  __syncthreads();
  if (tid < kMaxE) {
    int pre = 0;
    for (int w = 0; w < warp; ++w) pre += wsum[w];
    incl += pre;
    if (tid < E) {
      offs[tid] = incl - kept;
      if (rank == 0) {
        offsets[tid] = incl - kept;
        if (tid == E - 1) offsets[E] = incl;
      }
    }
  }
  __syncthreads();
  const unsigned lt = lanemask_lt();
#pragma unroll
  for (int it = 0; it < ITERS; ++it) {
    const long long a = s0 + it * 32 + lane;
    const int id = v[it];
    const unsigned m = __match_any_sync(0xffffffffu, id);
    int r = 0;
    if (id >= 0) r = cbase[id] + row[id] + __popc(m & lt);
    __syncwarp();
    if (id >= 0 && lane == __ffs(m) - 1) row[id] += __popc(m);
    __syncwarp();
    if (id >= 0) {
      int p = -1;
      if (cap < 0 || r < cap) {
        p = offs[id] + r;
        perm_to_assign[p] = (int32_t)a;
      }
      assign_to_perm[a] = p;
    } else if (a < A) {
      assign_to_perm[a] = -1;
    }
  }
  cluster_wait();  // every CTA of the cluster has finished reading this CTA's counts
}

template <int WARPS, int ITERS>
moe_status launch_cluster_permute(const int32_t* ids, long long A, int E, long long cap, int C,
                                  int32_t* counts, int32_t* offsets, int32_t* a2p, int32_t* p2a,
                                  unsigned* status, cudaStream_t st) {
  launch_begin(K_PERMUTE_CLUSTER, st);
  launch_kernel(permute_cluster_kernel<WARPS, ITERS>, dim3((unsigned)C), dim3(WARPS * 32), 0, st,
                (unsigned)C, ids, A, E, cap, C, counts, offsets, a2p, p2a, status);
  return launch_end(K_PERMUTE_CLUSTER, st);
}

}  // namespace

namespace {

// x_perm[p] = x[perm_to_assign[p] / K] for p < offsets[E]; 16-byte vectors. One warp moves
// a 2 KB segment (128 vectors) of one row: the row's source token is loaded once per lane
// and each lane keeps four independent 16-byte loads in flight. The rows are stored with an
// L2 evict-last policy: the kernel after this one reads them back (67 MB at the Mixtral
// shape fits in L2).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ p2a,
                                                          const int32_t* __restrict__ n_kept_ptr,
                                                          int K, int T, int vec_per_row,
                                                          uint4* __restrict__ x_perm,
                                                          unsigned* status) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const long long n_kept = *n_kept_ptr;
  const int segs = (vec_per_row + 127) / 128;
  const long long units = n_kept * segs;
  const int lane = threadIdx.x & 31;
  const uint64_t keep = l2_policy_evict_last();  // the next kernel reads the rows back
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long u = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units;
       u += warps) {
    const long long p = u / segs;
    const int v0 = (int)(u - p * segs) * 128 + lane;
    const int a = p2a[p];
    const int t = a / K;
    if (a < 0 || t >= T) {
      if (lane == 0) report(status, MOE_ERR_DEVICE_INDEX);
      continue;
    }
    const uint4* src = x + (size_t)t * vec_per_row;
    uint4* dst = x_perm + (size_t)p * vec_per_row;
    uint4 r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (v0 + 32 * j < vec_per_row) r[j] = src[v0 + 32 * j];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (v0 + 32 * j < vec_per_row) st_global_hint(dst + v0 + 32 * j, r[j], keep);
  }
}

}  // namespace

moe_status launch_gather_rows(const moe_shape& s, const void* x, const int32_t* p2a,
                              const int32_t* offsets, void* x_perm, cudaStream_t st);

size_t permute_scratch_bytes(const moe_shape& s) {
  const long long A = (long long)s.T * s.K;
  const long long nchunks = (A + kChunk - 1) / kChunk;
  return (size_t)(2 * nchunks * s.E) * sizeof(int32_t);
}

moe_status launch_permute(const moe_shape& s, const int32_t* ids, int32_t* counts,
                          int32_t* offsets, int32_t* a2p, int32_t* p2a, const void* x,
                          void* x_perm, void* scratch, cudaStream_t st) {
  const long long A = (long long)s.T * s.K;
  const int nchunks = (int)((A + kChunk - 1) / kChunk);
  int32_t* chunk_counts = (int32_t*)scratch;
  int32_t* chunk_base = chunk_counts + (size_t)nchunks * s.E;
  const long long cap =
      (s.capacity_factor > 0.f)
          ? (long long)ceil((double)s.capacity_factor * (double)s.T * (double)s.K / (double)s.E)
          : -1;
  unsigned* status = device_status_ptr();
  moe_status r;
  if (A > 0 && A <= kSmallMax) {
    launch_begin(K_PERMUTE_SMALL, st);
    launch_kernel(permute_small_kernel, dim3(1), dim3(kSmallWarps * 32), 0, st, 1, ids, A, s.E, cap,
                  counts, offsets, a2p, p2a, status);
    if ((r = launch_end(K_PERMUTE_SMALL, st)) != MOE_OK) return r;
  } else if (A > 0 && A <= kClusterMax) {
    // one cluster of <= 8 CTAs: 8-warp CTAs with 1, 2 or 4 groups of 32 ids per warp up to
    // 8192 assignments, 32-warp CTAs with 2 or 4 groups beyond
    int warps = 8, iters = 1;
    while ((long long)kClusterMaxCtas * warps * 32 * iters < A) {
      if (iters < 4) iters <<= 1;
      else {
        warps = 32;
        iters = 2;
      }
    }
    const int per_cta = warps * 32 * iters;
    const int C = (int)((A + per_cta - 1) / per_cta);
    if (warps == 8)
      r = iters == 1 ? launch_cluster_permute<8, 1>(ids, A, s.E, cap, C, counts, offsets, a2p, p2a, status, st)
        : iters == 2 ? launch_cluster_permute<8, 2>(ids, A, s.E, cap, C, counts, offsets, a2p, p2a, status, st)
                     : launch_cluster_permute<8, 4>(ids, A, s.E, cap, C, counts, offsets, a2p, p2a, status, st);
    else
      r = iters == 2 ? launch_cluster_permute<32, 2>(ids, A, s.E, cap, C, counts, offsets, a2p, p2a, status, st)
                     : launch_cluster_permute<32, 4>(ids, A, s.E, cap, C, counts, offsets, a2p, p2a, status, st);
    if (r != MOE_OK) return r;
  } else if (nchunks > 0) {
    launch_begin(K_HIST, st);
    launch_kernel(hist_kernel, dim3((unsigned)nchunks), dim3(kWarps * 32), 0, st, 1, ids, A, s.E,
                  chunk_counts, status);
    if ((r = launch_end(K_HIST, st)) != MOE_OK) return r;
    const int fused = (long long)nchunks * s.E <= kFusedScanMax;
    if (!fused) {
      int epad = 1;
      while (epad < s.E) epad <<= 1;
      launch_begin(K_SCAN, st);
      launch_kernel(scan_kernel, dim3(1), dim3(kScanThreads), 0, st, 1,
                    (const int32_t*)chunk_counts, chunk_base, nchunks, s.E, epad, cap, counts,
                    offsets);
      if ((r = launch_end(K_SCAN, st)) != MOE_OK) return r;
    }
    launch_begin(K_SCATTER, st);
    launch_kernel(scatter_kernel, dim3((unsigned)nchunks), dim3(kWarps * 32), 0, st, 1, ids, A,
                  s.E, cap, (const int32_t*)chunk_counts, (const int32_t*)chunk_base, nchunks,
                  fused, counts, offsets, a2p, p2a, status);
    if ((r = launch_end(K_SCATTER, st)) != MOE_OK) return r;
  }
  if (x != nullptr && x_perm != nullptr && A > 0)
    return launch_gather_rows(s, x, p2a, offsets, x_perm, st);
  return MOE_OK;
}

moe_status launch_gather_rows(const moe_shape& s, const void* x, const int32_t* p2a,
                              const int32_t* offsets, void* x_perm, cudaStream_t st) {
  const long long A = (long long)s.T * s.K;
  if (A == 0) return MOE_OK;
  const int elem = (s.dtype == MOE_BF16) ? 2 : 4;
  const int vec_per_row = s.d * elem / 16;
  const long long units = A * ((vec_per_row + 127) / 128);  // one warp each
  long long blocks = (units + 7) / 8;
  const long long cap_blocks = (long long)sm_count() * 8;
  if (blocks > cap_blocks) blocks = cap_blocks;
  launch_begin(K_GATHER, st);
  launch_kernel(gather_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, st, 1, (const uint4*)x,
                p2a, (const int32_t*)(offsets + s.E), s.K, s.T, vec_per_row, (uint4*)x_perm,
                device_status_ptr());
  return launch_end(K_GATHER, st);
}

// ------------------------------------------------------------------ token rounding
// Tile-aware token rounding (SonicMoE explainer, section 6.5; the rule is the library's
// reading, stated in moe.h). One CTA per expert e, after an uncapped permutation (its slots
// [offsets[e], offsets[e] + c) hold its c routed assignments in token order). Keys are
// (logit for e as an order-preserving 32-bit integer, +0 for both zeros) << 32 |
// (2^32 - 1 - t): ascending keys run from the weakest token up and every key is distinct.
// Rounding down drops the c mod R smallest keys of e's routed tokens; rounding up adds the
// m largest keys among the tokens that did not route to e. Both place a threshold with a
// radix select over the keys, cached in shared memory when they fit.
namespace {

// A threshold on the distinct 64-bit keys key_of(j) over the j < n for which key_of returns
// true, placed at the need-th smallest (1-based) of them, q: GE returns theta with
// {key >= theta} = {key >= q}; otherwise theta with {key <= theta} = {key <= q}. An 8-pass
// radix select, 8 bits a pass from the top, a 256-bin shared histogram, the bin found by
// warp 0's shuffle scan and ballot; it stops early once q's bin is known to lie wholly on
// the selected side (GE: q is the bin's smallest key; else its largest), which for
// continuous logits happens after two or three passes. Every thread of the NT-thread CTA
// calls it.
template <int NT, bool GE, typename KeyOf>
__device__ uint64_t radix_threshold(int n, int need, KeyOf key_of, unsigned* hist,
                                    unsigned long long* s_pre, int* s_need, int* s_done) {
  const int tid = threadIdx.x;
  uint64_t pre = 0;
  for (int d = 7; d >= 0; --d) {
    const uint64_t hi = d == 7 ? 0ull : (~0ull << (8 * (d + 1)));
    for (int b = tid; b < 256; b += NT) hist[b] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += NT) {
      uint64_t key;
      if (key_of(j, key) && ((key ^ pre) & hi) == 0) atomicAdd(&hist[(key >> (8 * d)) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {  // warp 0: the bin where the running count reaches `need`
      const int lane = tid;
      unsigned v[8], ls = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[q] = hist[lane * 8 + q];
        ls += v[q];
      }
      unsigned incl = ls;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned excl = incl - ls;
      const unsigned hit = __ballot_sync(0xffffffffu, excl < (unsigned)need && incl >= (unsigned)need);
      if (lane == __ffs(hit) - 1) {
        unsigned run = excl, cnt = v[7];
        int b = lane * 8 + 7;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (run + v[q] >= (unsigned)need) {
            b = lane * 8 + q;
            cnt = v[q];
            break;
          }
          run += v[q];
        }
        const int nn = need - (int)run;  // q's rank inside bin b
        uint64_t p = pre | ((uint64_t)b << (8 * d));
        const bool done = d == 0 || (GE ? nn == 1 : nn == (int)cnt);
        if (done && !GE && d > 0) p |= (1ull << (8 * d)) - 1;  // every lower digit at its top
        *s_need = nn;
        *s_pre = p;
        *s_done = done;
      }
    }
    __syncthreads();
    pre = *s_pre;
    need = *s_need;
    const bool done = *s_done;
    __syncthreads();
    if (done) break;
  }
  return pre;
}

// Threads of the selection kernel: its loops are latency-bound with one CTA per expert.
constexpr int kRoundThreads = 1024;

// Rounding up or to the nearest tile: the tokens expert e gains, as a count, from its routed
// count c (0 when it rounds down or is whole).
__device__ __forceinline__ int round_adds(int c, int R, int mode, int T) {
  const int r = c % R;
  if (r == 0 || !(mode == 1 || (mode == 2 && r > R - r))) return 0;
  return min(R - r, T - c);
}

__device__ __forceinline__ uint32_t ord_logit(float v) {
  if (v == 0.f) v = 0.f;  // -0 and +0 are one value
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // ascending order of the floats
}

// Writes the extended id list ids_ext [T*K + NA] whole (NA = 0 when only rounding down).
// Each CTA writes its expert's routed entries: e, or -1 for those an expert that rounds
// down drops. An expert that rounds up (mode 1, or 2 with r > R - r) gains the m =
// min(R - r, T - c) strongest tokens that did not route to it (a shared bitmap marks its
// routed ones); they are written in ascending order to add_tok[base ...] and as e into
// ids_ext[T*K + base ...], base = the tokens gained by the experts before e. CTA 0 sets the
// unused tail of both added lists to -1. The keys live in the dynamic shared memory (cap
// bytes) when they fit: 32 bits a token when rounding up (the token is the index), 64 bits
// a routed slot when rounding down.
__global__ void __launch_bounds__(kRoundThreads) round_select_kernel(
    const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets0,
    const int32_t* __restrict__ p2a0, const float* __restrict__ logits, int T, int K, int E,
    int R, int mode, int NA, int cap, int32_t* __restrict__ ids_ext,
    int32_t* __restrict__ add_tok) {
  extern __shared__ __align__(16) uint8_t round_cache[];
  __shared__ uint32_t routed[kRoundUpMaxTokens / 32];
  __shared__ unsigned hist[256];
  __shared__ unsigned long long s_pre;
  __shared__ int s_need, s_base, s_total, s_done;
  __shared__ int wsum[kRoundThreads / 32];
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t A0 = (size_t)T * K;
  const int c = counts[e];
  const int r = c % R;
  const int off = offsets0[e];
  if (NA > 0) {
    if (tid == 0) s_base = s_total = 0;
    __syncthreads();
    for (int i = tid; i < E; i += kRoundThreads) {
      const int v = round_adds(counts[i], R, mode, T);
      if (i < e) atomicAdd(&s_base, v);
      atomicAdd(&s_total, v);
    }
    __syncthreads();
    if (e == 0)
      for (int j = s_total + tid; j < NA; j += kRoundThreads) {
        ids_ext[A0 + j] = -1;
        add_tok[j] = -1;
      }
  }
  const bool up = NA > 0 && r != 0 && (mode == 1 || (mode == 2 && r > R - r));
  if (!up) {
    if (r == 0 || c < R) {  // whole tiles, or too few to drop: every routed entry stays
      for (int j = tid; j < c; j += kRoundThreads) ids_ext[p2a0[off + j]] = e;
      return;
    }
    uint64_t* kc = reinterpret_cast<uint64_t*>(round_cache);
    const bool cached = (long long)c * 8 <= cap;  // uniform across the CTA
    if (cached) {
      for (int j = tid; j < c; j += kRoundThreads) {
        const int t = p2a0[off + j] / K;
        kc[j] = ((uint64_t)ord_logit(logits[(size_t)t * E + e]) << 32) |
                (uint64_t)(0xffffffffu - (uint32_t)t);
      }
      __syncthreads();
    }
    auto key_of = [&](int j, uint64_t& key) {
      if (cached) {
        key = kc[j];
      } else {
        const int t = p2a0[off + j] / K;
        key = ((uint64_t)ord_logit(logits[(size_t)t * E + e]) << 32) |
              (uint64_t)(0xffffffffu - (uint32_t)t);
      }
      return true;
    };
    // the r-th smallest key: it and every smaller one are dropped
    const uint64_t pre = radix_threshold<kRoundThreads, false>(c, r, key_of, hist, &s_pre, &s_need, &s_done);
    for (int j = tid; j < c; j += kRoundThreads) {
      uint64_t key;
      key_of(j, key);
      ids_ext[p2a0[off + j]] = key <= pre ? -1 : e;
    }
    return;
  }
  const int base = s_base;
  const int m = min(R - r, T - c);
  for (int i = tid; i < T / 32 + 1 && i < kRoundUpMaxTokens / 32; i += kRoundThreads) routed[i] = 0;
  uint32_t* uc = reinterpret_cast<uint32_t*>(round_cache);
  const bool cached = (long long)T * 4 <= cap;  // uniform across the CTA
  if (cached)
    for (int t = tid; t < T; t += kRoundThreads) uc[t] = ord_logit(logits[(size_t)t * E + e]);
  __syncthreads();
  for (int j = tid; j < c; j += kRoundThreads) {
    const int a = p2a0[off + j];
    ids_ext[a] = e;
    const int t = a / K;
    atomicOr(&routed[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  if (m <= 0) return;
  auto key_of = [&](int t, uint64_t& key) {
    if ((routed[t >> 5] >> (t & 31)) & 1u) return false;
    const uint32_t u = cached ? uc[t] : ord_logit(logits[(size_t)t * E + e]);
    key = ((uint64_t)u << 32) | (uint64_t)(0xffffffffu - (uint32_t)t);
    return true;
  };
  // the m-th largest of the T - c candidate keys = their (T - c - m + 1)-th smallest
  const uint64_t theta =
      radix_threshold<kRoundThreads, true>(T, T - c - m + 1, key_of, hist, &s_pre, &s_need, &s_done);
  // the chosen tokens in ascending order, kRoundThreads at a time
  int run = 0;
  for (int t0 = 0; t0 < T; t0 += kRoundThreads) {
    const int t = t0 + tid;
    uint64_t key = 0;
    const bool chosen = t < T && key_of(t, key) && key >= theta;
    const unsigned bal = __ballot_sync(0xffffffffu, chosen);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int before = run, total = 0;
    for (int w = 0; w < kRoundThreads / 32; ++w) {
      if (w < warp) before += wsum[w];
      total += wsum[w];
    }
    if (chosen) {
      const int pos = base + before + __popc(bal & lanemask_lt());
      add_tok[pos] = t;
      ids_ext[A0 + pos] = e;
    }
    run += total;
    __syncthreads();
  }
}

// Token-major lists of the added assignments, in one CTA of 1024 threads whose phases are
// separated by block barriers (a few thousand entries):
//   1. per-token counts of the added assignments (atomics on zeroed counters);
//   2. add_ptr = their exclusive scan (each thread a contiguous run of tokens, the runs'
//      sums scanned across the block); the counters are zeroed again;
//   3. each added assignment into its token's list at an atomic cursor (any order; the
//      finishing kernel sorts each list).
__global__ void __launch_bounds__(1024) round_lists_kernel(const int32_t* __restrict__ ids_add,
                                                           const int32_t* __restrict__ add_tok,
                                                           int NA, int T, int32_t* cnt,
                                                           int32_t* add_ptr, int32_t* add_idx,
                                                           unsigned* status) {
  __shared__ int wsum[32];
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int t = tid; t < T; t += 1024) cnt[t] = 0;
  __syncthreads();
  for (int j = tid; j < NA; j += 1024) {  // 1. counts
    if (ids_add[j] < 0) continue;
    const int t = add_tok[j];
    if (t < 0 || t >= T) {
      report(status, MOE_ERR_DEVICE_INDEX);
      continue;
    }
    atomicAdd(&cnt[t], 1);
  }
  __syncthreads();
  {  // 2. exclusive scan
    const int per = (T + 1023) / 1024;
    const int b = tid * per, e = min(T, b + per);
    int sum = 0;
    for (int t = b; t < e; ++t) sum += cnt[t];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = wsum[lane];
      int iv = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, iv, o);
        if (lane >= o) iv += y;
      }
      wsum[lane] = iv - v;
    }
    __syncthreads();
    int run = wsum[warp] + incl - sum;
    for (int t = b; t < e; ++t) {
      add_ptr[t] = run;
      run += cnt[t];
      cnt[t] = 0;
    }
    if (tid == 1023) add_ptr[T] = run;
  }
  __syncthreads();
  for (int j = tid; j < NA; j += 1024) {  // 3. fill
    if (ids_add[j] < 0) continue;
    const int t = add_tok[j];
    if (t < 0 || t >= T) continue;
    add_idx[add_ptr[t] + atomicAdd(&cnt[t], 1)] = j;
  }
  __syncthreads();
}

// The rest of rounding up, one thread per entry over max(T, n_kept) (both independent):
//   p < n_kept: the token of expert-major slot p (a < T*K is token a / K, an added
//     a = T*K + j is add_tok[j]);
//   t < T with added assignments: its list sorted ascending (= expert order), then,
//     renormalised, w = exp(l - l_top) / (sum over the K routed and the added of
//     exp(l_j - l_top)) summed in slot order then list order, l_top the logit of its first
//     routed expert (the largest); plain softmax: the added ones get softmax(l) over all E,
//     the routed ones keep theirs.
__global__ void __launch_bounds__(256) round_finish_kernel(
    const int32_t* __restrict__ p2a, const int32_t* __restrict__ n_kept_ptr, int T, int K, int E,
    int renorm, const float* __restrict__ logits, const int32_t* __restrict__ ids,
    const int32_t* __restrict__ ids_add, const int32_t* __restrict__ add_tok,
    const int32_t* __restrict__ add_ptr, int32_t* __restrict__ add_idx,
    int32_t* __restrict__ slot_tok, float* __restrict__ topk_w, float* __restrict__ add_w) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const int n_kept = *n_kept_ptr;
  const long long A0 = (long long)T * K;
  const int n = max(n_kept, T);
  for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) {
    if (i < n_kept) {
      const long long a = p2a[i];
      slot_tok[i] = a < A0 ? (int32_t)(a / K) : add_tok[a - A0];
    }
    if (i >= T) continue;
    const int t = i;
    const int lo = add_ptr[t], hi = add_ptr[t + 1];
    if (hi == lo) continue;
    for (int q = lo + 1; q < hi; ++q) {  // insertion sort (a token gains a few at most)
      const int v = add_idx[q];
      int k = q - 1;
      while (k >= lo && add_idx[k] > v) {
        add_idx[k + 1] = add_idx[k];
        --k;
      }
      add_idx[k + 1] = v;
    }
    const float* lg = logits + (size_t)t * E;
    const float top = lg[ids[(size_t)t * K]];
    float den = 0.f;
    if (renorm) {
      for (int k = 0; k < K; ++k) den += expf(lg[ids[(size_t)t * K + k]] - top);
      for (int q = lo; q < hi; ++q) den += expf(lg[ids_add[add_idx[q]]] - top);
      for (int k = 0; k < K; ++k)
        topk_w[(size_t)t * K + k] = expf(lg[ids[(size_t)t * K + k]] - top) / den;
    } else {  // the plain softmax over all E (the top logit is the maximum)
      for (int q = 0; q < E; ++q) den += expf(lg[q] - top);
    }
    for (int q = lo; q < hi; ++q) add_w[add_idx[q]] = expf(lg[ids_add[add_idx[q]]] - top) / den;
  }
}

}  // namespace

// Dynamic shared memory of the selection kernel: up to 192 KB of cached keys (8 bytes a
// token bounds both directions), beside its 17 KB of static arrays.
constexpr int kRoundCacheMax = 192 * 1024;

moe_status launch_round_select_kernel(const moe_shape& s, const int32_t* counts,
                                      const int32_t* offsets0, const int32_t* p2a0,
                                      const float* logits, int mode, int NA, int32_t* ids_ext,
                                      int32_t* add_tok, cudaStream_t st) {
  const int cap = (int)std::min<long long>(kRoundCacheMax, (long long)s.T * 8);
  if (cudaFuncSetAttribute(round_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kRoundCacheMax) != cudaSuccess)
    return MOE_ERR_CUDA;
  launch_begin(K_TILE_ROUND, st);
  launch_kernel(round_select_kernel, dim3((unsigned)s.E), dim3(kRoundThreads), (size_t)cap, st, 1, counts,
                offsets0, p2a0, logits, s.T, s.K, s.E, s.tile_round, mode, NA, cap, ids_ext,
                add_tok);
  return launch_end(K_TILE_ROUND, st);
}

moe_status launch_permute_rounded(const moe_shape& s, const int32_t* ids, const float* logits,
                                  int32_t* counts, int32_t* offsets, int32_t* a2p, int32_t* p2a,
                                  const void* x, void* x_perm, void* scratch, int32_t* round_ids,
                                  int32_t* round_counts, cudaStream_t st) {
  moe_status r;
  // 1. uncapped permutation: raw counts, each expert's assignments in token order
  if ((r = launch_permute(s, ids, counts, offsets, a2p, p2a, nullptr, nullptr, scratch, st)) !=
      MOE_OK)
    return r;
  // 2. the ids again, with the rounded-away assignments set to -1
  if ((r = launch_round_select_kernel(s, counts, offsets, p2a, logits, 0, 0, round_ids, nullptr,
                                      st)) != MOE_OK)
    return r;
  // 3. the final permutation of what is kept (its counts are the kept ones: not returned)
  return launch_permute(s, round_ids, round_counts, offsets, a2p, p2a, x, x_perm, scratch, st);
}

moe_status launch_round_select(const moe_shape& s, const int32_t* counts, const int32_t* offsets0,
                               const int32_t* p2a0, const float* logits, int32_t* ids_ext,
                               int32_t* add_tok, cudaStream_t st) {
  if (s.T > kRoundUpMaxTokens) return MOE_ERR_UNSUPPORTED;
  return launch_round_select_kernel(s, counts, offsets0, p2a0, logits, s.tile_round_mode,
                                    s.E * (s.tile_round - 1), ids_ext, add_tok, st);
}

moe_status launch_round_lists(const moe_shape& s, const int32_t* ids_add, const int32_t* add_tok,
                              int32_t* cursor, int32_t* add_ptr, int32_t* add_idx,
                              cudaStream_t st) {
  launch_begin(K_TILE_ROUND, st);
  launch_kernel(round_lists_kernel, dim3(1), dim3(1024), 0, st, 1, ids_add, add_tok,
                s.E * (s.tile_round - 1), s.T, cursor, add_ptr, add_idx, device_status_ptr());
  return launch_end(K_TILE_ROUND, st);
}

moe_status launch_round_finish(const moe_shape& s, const int32_t* p2a, const int32_t* offsets,
                               const float* logits, const int32_t* ids, const int32_t* ids_add,
                               const int32_t* add_tok, const int32_t* add_ptr, int32_t* add_idx,
                               int32_t* slot_tok, float* topk_w, float* add_w, cudaStream_t st) {
  const long long A = (long long)s.T * s.K + (long long)s.E * (s.tile_round - 1);
  long long blocks = (std::max<long long>(A, s.T) + 255) / 256;
  if (blocks > (long long)sm_count() * 8) blocks = (long long)sm_count() * 8;
  launch_begin(K_TILE_ROUND, st);
  launch_kernel(round_finish_kernel, dim3((unsigned)blocks), dim3(256), 0, st, 1, p2a,
                offsets + s.E, s.T, s.K, s.E, s.renormalize, logits, ids, ids_add, add_tok,
                add_ptr, add_idx, slot_tok, topk_w, add_w);
  return launch_end(K_TILE_ROUND, st);
}

// ------------------------------------------------------------------ no-allocation variant
// For callers that may not allocate device memory while they run: a serving engine that
// plans its whole memory budget at start-up and forbids allocation on the request path, an
// embedded runtime with a fixed arena, or code that runs where cudaMalloc would synchronise
// the device. Their permute scratch lives in this file-scope device array instead of a
// caller workspace. Every GPU that loads the library holds it until the process exits.
// All calls share it and it keeps the last call's contents. Problems of up to kClusterMax
// assignments (one CTA or one cluster) use none of it; larger ones use the per-chunk
// counts, written by the histogram kernel before the scan or the scatter reads them, and,
// when the scan is not fused into the scatter, the rank bases, written by the scan kernel
// before the scatter reads them: nothing in it has to start at zero. Calls whose kernels
// overlap on the GPU (different streams, or several host threads) race on it and must be
// serialised by the caller.
static __device__ __align__(256) unsigned char g_permute_static_scratch[kPermuteStaticScratchBytes];

namespace {
std::mutex g_static_mu;
void* g_static_ptr[64];  // device address of the array, per device
}  // namespace

// Device address of the static scratch on the current device. The first call on a device
// resolves it with cudaGetSymbolAddress (with that device current); later calls reuse it
// (it stays valid until the device is reset, which the library does not support).
static moe_status static_scratch_ptr(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_static_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return MOE_OK;
}

moe_status launch_permute_static(const moe_shape& s, const int32_t* ids, int32_t* counts,
                                 int32_t* offsets, int32_t* a2p, int32_t* p2a, const void* x,
                                 void* x_perm, cudaStream_t st) {
  if (permute_scratch_bytes(s) > (size_t)kPermuteStaticScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const moe_status r = static_scratch_ptr(&scratch);
  if (r != MOE_OK) return r;
  return launch_permute(s, ids, counts, offsets, a2p, p2a, x, x_perm, scratch, st);
}

}  // namespace moe
