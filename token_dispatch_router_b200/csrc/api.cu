// C ABI of the MoE-layer forward: argument checks, workspace layout, the device status
// word, the opt-in profiler and the entry points declared in include/moe.h.
#include <math.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "common.cuh"
#include "round.cuh"

namespace moe {

moe_status launch_route(const moe_shape& s, const void* x, const void* w_r, const float* bias,
                        const float* logits_in, float* logits_out, int32_t* ids, float* w,
                        cudaStream_t st);
size_t permute_scratch_bytes(const moe_shape& s);
moe_status launch_permute(const moe_shape& s, const int32_t* ids, int32_t* counts,
                          int32_t* offsets, int32_t* a2p, int32_t* p2a, const void* x,
                          void* x_perm, void* scratch, cudaStream_t st);
moe_status launch_ffn_simt(const moe_shape& s, const void* x, const int32_t* offsets,
                           const int32_t* p2a, const void* w_gate, const void* w_up,
                           const void* w_down, void* a_act, void* y_perm, cudaStream_t st);
moe_status launch_combine(const moe_shape& s, const void* y_perm, const int32_t* a2p,
                          const float* topk_w, void* out, cudaStream_t st);
moe_status launch_selftest_timeout(uint64_t limit_ns, cudaStream_t st);
bool route_tc_supported(const moe_shape& s);
moe_status launch_ffn_tc_mixed(const moe_shape& s, const void* x, const int32_t* offsets,
                               const int32_t* p2a, const void* w_gate, const void* w_up,
                               const void* w_down, void* a_act, void* y_perm, int gateup_mode,
                               bool pair_down, void* h_out, cudaStream_t st);
size_t backward_scratch_bytes(const moe_shape& s, bool with_dx);
moe_status launch_router_backward(const moe_shape& s, const void* x, const void* w_r,
                                  const float* logits, const int32_t* ids, const float* topk_w,
                                  const float* d_w, float* d_logits, float* d_w_r,
                                  float* d_bias, void* d_x, cudaStream_t st);
moe_status launch_backward(const moe_shape& s, const void* d_out, const float* topk_w,
                           const int32_t* offsets, const int32_t* p2a, const int32_t* a2p,
                           const void* w_gate, const void* w_up, const void* w_down,
                           const void* h, void* d_h, float* d_w, void* d_x, void* scratch,
                           cudaStream_t st);
moe_status launch_permute_static(const moe_shape& s, const int32_t* ids, int32_t* counts,
                                 int32_t* offsets, int32_t* a2p, int32_t* p2a, const void* x,
                                 void* x_perm, cudaStream_t st);
moe_status launch_route_tc(const moe_shape& s, const void* x, const void* w_r, const float* bias,
                           float* logits_out, int32_t* ids, float* w, cudaStream_t st);
moe_status launch_gather_rows(const moe_shape& s, const void* x, const int32_t* p2a,
                              const int32_t* offsets, void* x_perm, cudaStream_t st);
moe_status launch_permute_rounded(const moe_shape& s, const int32_t* ids, const float* logits,
                                  int32_t* counts, int32_t* offsets, int32_t* a2p, int32_t* p2a,
                                  const void* x, void* x_perm, void* scratch, int32_t* round_ids,
                                  int32_t* round_counts, cudaStream_t st);

moe_status launch_round_select(const moe_shape& s, const int32_t* counts, const int32_t* offsets0,
                               const int32_t* p2a0, const float* logits, int32_t* ids_ext,
                               int32_t* add_tok, cudaStream_t st);
moe_status launch_round_lists(const moe_shape& s, const int32_t* ids_add, const int32_t* add_tok,
                              int32_t* cursor, int32_t* add_ptr, int32_t* add_idx,
                              cudaStream_t st);
moe_status launch_round_finish(const moe_shape& s, const int32_t* p2a, const int32_t* offsets,
                               const float* logits, const int32_t* ids, const int32_t* ids_add,
                               const int32_t* add_tok, const int32_t* add_ptr, int32_t* add_idx,
                               int32_t* slot_tok, float* topk_w, float* add_w, cudaStream_t st);
moe_status launch_combine_added(const moe_shape& s, const void* y_perm, const int32_t* a2p,
                                const float* topk_w, void* out, const int32_t* add_ptr,
                                const int32_t* add_idx, const float* add_w, long long n_rows,
                                cudaStream_t st);

// Rounding up or to the nearest tile: added assignments beyond T * K.
bool rounds_up(const moe_shape& s) { return s.tile_round > 1 && s.tile_round_mode != 0; }
// The permutation over the extended assignment list runs as T * K + E * (R - 1)
// one-assignment "tokens".
moe_shape ext_shape(const moe_shape& s) {
  moe_shape e = s;
  e.T = s.T * s.K + s.E * (s.tile_round - 1);
  e.K = 1;
  e.capacity_factor = 0.f;
  e.tile_round = 0;
  e.tile_round_mode = 0;
  return e;
}

// ------------------------------------------------------------------ device state
__device__ unsigned int g_device_status;

namespace {
constexpr int kMaxDev = 64;
unsigned int* g_status_ptr[kMaxDev];
int g_sms[kMaxDev];
std::mutex g_dev_mu;

int cur_dev() {
  int d = 0;
  cudaGetDevice(&d);
  return (d >= 0 && d < kMaxDev) ? d : 0;
}
}  // namespace

unsigned int* device_status_ptr() {
  const int d = cur_dev();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_status_ptr[d] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) == cudaSuccess) g_status_ptr[d] = (unsigned*)p;
  }
  return g_status_ptr[d];
}

int sm_count() {
  const int d = cur_dev();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_sms[d] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    g_sms[d] = n > 0 ? n : 1;
  }
  return g_sms[d];
}

// ------------------------------------------------------------------ profiler
namespace {
const char* kKernelNames[K_COUNT] = {
    "route",        "hist",          "scan",           "scatter",     "gather_rows", "gateup_tc",
    "down_tc",      "gateup_simt",   "down_simt",      "combine",     "selftest_timeout",
    "route_tc",     "permute_small", "gateup_tc2",   "down_tc2",
    "permute_cluster", "tile_round", "bwd_act", "bwd_dw", "bwd_dx",
    "router_dlogits", "router_dwr", "router_dx", "omni_logits", "omni_topk", "omni_count",
    "omni_scan", "omni_scatter", "omni_sort", "omni_act", "omni_out"};

struct ProfRec {
  int kid;
  cudaEvent_t a, b;
};
bool g_prof_on = false;
std::vector<ProfRec> g_recs;
std::vector<cudaEvent_t> g_pool;
long long g_launches = 0;
std::mutex g_prof_mu;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

void launch_begin(int kid, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ++g_launches;
  if (!g_prof_on) return;
  ProfRec r{kid, take_event(), take_event()};
  cudaEventRecord(r.a, s);
  g_recs.push_back(r);
}

moe_status launch_end(int kid, cudaStream_t s) {
  const cudaError_t err = cudaGetLastError();
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (g_prof_on && !g_recs.empty() && g_recs.back().kid == kid) cudaEventRecord(g_recs.back().b, s);
  }
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ------------------------------------------------------------------ checks and layout
namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int elem_bytes(const moe_shape& s) { return s.dtype == MOE_BF16 ? 2 : 4; }

moe_status check_shape(const moe_shape* s, bool need_d, bool need_ffn) {
  if (s == nullptr) return MOE_ERR_INVALID_ARG;
  if (s->dtype != MOE_F32 && s->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->E < 1 || s->K < 1 || s->K > s->E) return MOE_ERR_INVALID_ARG;
  if (s->E > 256 || s->K > 32) return MOE_ERR_UNSUPPORTED;
  if ((long long)s->T * s->K > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (isnan(s->capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (s->tile_round < 0 || (s->tile_round > 0 && s->capacity_factor > 0.f))
    return MOE_ERR_INVALID_ARG;  // token rounding and a capacity limit are exclusive
  if (s->tile_round_mode < 0 || s->tile_round_mode > 2) return MOE_ERR_INVALID_ARG;
  if (rounds_up(*s)) {  // added assignments: E * (R - 1) beyond T * K, int32 indices
    if ((long long)s->T * s->K + (long long)s->E * (s->tile_round - 1) > 0x7fffffffLL)
      return MOE_ERR_UNSUPPORTED;
    if (s->T > kRoundUpMaxTokens) return MOE_ERR_UNSUPPORTED;
  }
  if (s->ffn_variant < 0 || s->ffn_variant > 3) return MOE_ERR_INVALID_ARG;
  if (s->route_topk < 0 || s->route_topk > 2) return MOE_ERR_INVALID_ARG;
  if (need_d) {
    if (s->d < 64 || s->d % 64 != 0) return MOE_ERR_INVALID_ARG;
  }
  if (need_ffn) {
    const int nq = s->dtype == MOE_BF16 ? 64 : 16;
    if (s->n < nq || s->n % nq != 0) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

bool layout_of(const moe_shape& s, moe_workspace_layout* L) {
  const size_t T = (size_t)s.T, E = (size_t)s.E, K = (size_t)s.K;
  const bool up = rounds_up(s);
  const size_t NA = up ? E * (size_t)(s.tile_round - 1) : 0;  // added assignments at most
  const size_t A = T * K + NA;                                 // entries of both maps
  const size_t eb = (size_t)elem_bytes(s);
  size_t o = 0;
  L->logits = o;
  o = align256(o + T * E * 4);
  L->topk_ids = o;
  o = align256(o + A * 4);
  L->topk_w = o;
  o = align256(o + A * 4);
  L->counts = o;
  o = align256(o + E * 4);
  L->offsets = o;
  o = align256(o + (E + 1) * 4);
  L->assign_to_perm = o;
  o = align256(o + A * 4);
  L->perm_to_assign = o;
  o = align256(o + A * 4);
  L->permute_scratch = o;
  o = align256(o + permute_scratch_bytes(up ? ext_shape(s) : s));
  L->a_act = o;
  o = align256(o + A * (size_t)s.n * eb);
  L->y_perm = o;
  o = align256(o + A * (size_t)s.d * eb);
  L->round_ids = o;
  if (s.tile_round > 0) o = align256(o + A * 4);
  L->round_counts = o;
  if (s.tile_round > 0) o = align256(o + E * 4);
  L->add_tok = o;
  if (up) o = align256(o + NA * 4);
  L->add_w = o;
  if (up) o = align256(o + NA * 4);
  L->add_ptr = o;
  if (up) o = align256(o + (T + 1) * 4);
  L->add_idx = o;
  if (up) o = align256(o + NA * 4);
  L->add_cursor = o;
  if (up) o = align256(o + T * 4);
  L->slot_token = o;
  if (up) o = align256(o + A * 4);
  L->n_assign = A;
  L->total = o;
  return true;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// Tile variant (moe_shape.ffn_variant). Automatic choice, from measurements on B200: the
// gate/up GEMM runs single-CTA tiles (its gathered A operand gains nothing from pairing, and
// 256-row tiles pad twice as many rows); the down GEMM runs on CTA pairs once experts
// average at least 512 rows, where the pair's deeper pipeline beats the extra padding.
bool use_pair_down(const moe_shape& s) {
  if (s.ffn_variant != 0) return s.ffn_variant >= 2;
  return (long long)s.T * s.K >= 512LL * s.E;
}
int gateup_mode(const moe_shape& s) { return s.ffn_variant == 2 ? 1 : s.ffn_variant == 3 ? 2 : 0; }

}  // namespace
}  // namespace moe

namespace moe {
namespace {
// The layer forward with token rounding up or to the nearest tile (reading in moe.h).
// 1. route; 2. the uncapped permutation (raw counts, each expert's assignments in token
// order); 3. the extended id list: the routed ids, less those an expert that rounds down
// drops, then E * (R - 1) entries holding the added assignments' experts (-1 past the
// last); 4. the permutation
// of the extended list as T * K + E * (R - 1) one-assignment rows; 5. the token-major lists
// of the added assignments and the weights over each enlarged selection; 6. the token of
// every expert-major slot; 7. the grouped FFN over those rows; 8. combine with the added
// slots.
moe_status launch_forward_rounded_up(const moe_shape& s, const void* x, const void* w_r,
                                     const float* bias, const float* logits_in,
                                     const void* w_gate, const void* w_up, const void* w_down,
                                     void* out, uint8_t* ws, const moe_workspace_layout& L,
                                     bool pair_down, int gateup_mode, cudaStream_t st) {
  float* logits = (float*)(ws + L.logits);
  int32_t* ids = (int32_t*)(ws + L.topk_ids);
  float* w = (float*)(ws + L.topk_w);
  int32_t* counts = (int32_t*)(ws + L.counts);
  int32_t* offsets = (int32_t*)(ws + L.offsets);
  int32_t* a2p = (int32_t*)(ws + L.assign_to_perm);
  int32_t* p2a = (int32_t*)(ws + L.perm_to_assign);
  int32_t* ids_ext = (int32_t*)(ws + L.round_ids);
  int32_t* add_tok = (int32_t*)(ws + L.add_tok);
  int32_t* slot_tok = (int32_t*)(ws + L.slot_token);
  const size_t A0 = (size_t)s.T * s.K, NA = (size_t)s.E * (s.tile_round - 1);
  moe_status r;
  if ((r = moe_route(&s, x, w_r, bias, logits_in, logits, ids, w, (moe_stream_t)st)) != MOE_OK)
    return r;
  if ((r = launch_permute(s, ids, counts, offsets, a2p, p2a, nullptr, nullptr,
                          ws + L.permute_scratch, st)) != MOE_OK)
    return r;
  if ((r = launch_round_select(s, counts, offsets, p2a, logits, ids_ext, add_tok, st)) != MOE_OK)
    return r;
  const moe_shape xs = ext_shape(s);
  if ((r = launch_permute(xs, ids_ext, (int32_t*)(ws + L.round_counts), offsets, a2p, p2a,
                          nullptr, nullptr, ws + L.permute_scratch, st)) != MOE_OK)
    return r;
  int32_t* add_ptr = (int32_t*)(ws + L.add_ptr);
  int32_t* add_idx = (int32_t*)(ws + L.add_idx);
  if ((r = launch_round_lists(s, ids_ext + A0, add_tok, (int32_t*)(ws + L.add_cursor), add_ptr,
                              add_idx, st)) != MOE_OK)
    return r;
  if ((r = launch_round_finish(s, p2a, offsets, logits, ids, ids_ext + A0, add_tok, add_ptr,
                               add_idx, slot_tok, w, (float*)(ws + L.add_w), st)) != MOE_OK)
    return r;
  // the grouped FFN sees the extended list as one-assignment rows whose token is slot_tok[p]
  r = s.dtype == MOE_BF16 ? launch_ffn_tc_mixed(xs, x, offsets, slot_tok, w_gate, w_up, w_down,
                                                ws + L.a_act, ws + L.y_perm, gateup_mode,
                                                pair_down, nullptr, st)
                          : launch_ffn_simt(xs, x, offsets, slot_tok, w_gate, w_up, w_down,
                                            ws + L.a_act, ws + L.y_perm, st);
  if (r != MOE_OK) return r;
  return launch_combine_added(s, ws + L.y_perm, a2p, w, out, add_ptr, add_idx,
                              (const float*)(ws + L.add_w), (long long)(A0 + NA), st);
}

moe_status forward_impl(const moe_shape* s, const void* x, const void* w_r, const float* bias,
                        const float* logits_in, const void* w_gate, const void* w_up,
                        const void* w_down, void* out, void* h_out, void* workspace,
                        size_t ws_bytes, moe_stream_t stream) {
  moe_status r = check_shape(s, true, true);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!x || (!w_r && !logits_in) || !w_gate || !w_up || !w_down || !out) return MOE_ERR_INVALID_ARG;
  moe_workspace_layout L;
  layout_of(*s, &L);
  if (workspace == nullptr || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255) != 0) return MOE_ERR_INVALID_ARG;
  uint8_t* ws = (uint8_t*)workspace;
  const cudaStream_t st = (cudaStream_t)stream;
  float* logits = (float*)(ws + L.logits);
  int32_t* ids = (int32_t*)(ws + L.topk_ids);
  float* w = (float*)(ws + L.topk_w);
  int32_t* counts = (int32_t*)(ws + L.counts);
  int32_t* offsets = (int32_t*)(ws + L.offsets);
  int32_t* a2p = (int32_t*)(ws + L.assign_to_perm);
  int32_t* p2a = (int32_t*)(ws + L.perm_to_assign);
  if (rounds_up(*s)) {  // added assignments: the extended path
    if (h_out != nullptr) return MOE_ERR_UNSUPPORTED;
    if (s->dtype == MOE_BF16 &&
        (!aligned16(x) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down)))
      return MOE_ERR_INVALID_ARG;
    return launch_forward_rounded_up(*s, x, w_r, bias, logits_in, w_gate, w_up, w_down, out, ws,
                                     L, use_pair_down(*s), gateup_mode(*s), st);
  }
  if (s->tile_round > 0) {
    if ((r = moe_route(s, x, w_r, bias, logits_in, logits, ids, w, stream)) != MOE_OK) return r;
    if ((r = launch_permute_rounded(*s, ids, logits, counts, offsets, a2p, p2a, nullptr, nullptr,
                                    ws + L.permute_scratch, (int32_t*)(ws + L.round_ids),
                                    (int32_t*)(ws + L.round_counts), st)) != MOE_OK)
      return r;
  } else {
    if ((r = moe_route(s, x, w_r, bias, logits_in, logits, ids, w, stream)) != MOE_OK) return r;
    if ((r = launch_permute(*s, ids, counts, offsets, a2p, p2a, nullptr, nullptr,
                            ws + L.permute_scratch, st)) != MOE_OK)
      return r;
  }
  if (h_out != nullptr) {  // keep the gate/up pre-activations (single-CTA gate/up tiles)
    if (!aligned16(x) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down))
      return MOE_ERR_INVALID_ARG;
    r = launch_ffn_tc_mixed(*s, x, offsets, p2a, w_gate, w_up, w_down, ws + L.a_act,
                            ws + L.y_perm, 0, use_pair_down(*s), h_out, st);
  } else {
    r = moe_grouped_ffn(s, x, offsets, p2a, w_gate, w_up, w_down, ws + L.a_act, ws + L.y_perm,
                        stream);
  }
  if (r != MOE_OK) return r;
  return launch_combine(*s, ws + L.y_perm, a2p, w, out, st);
}
}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_permute_workspace_size(const moe_shape* s) {
  if (check_shape(s, false, false) != MOE_OK) return 0;
  size_t bytes = align256(permute_scratch_bytes(*s));
  if (s->tile_round > 0)  // the rounded ids and the kept counts (moe_dispatch)
    bytes += align256((size_t)s->T * s->K * 4) + align256((size_t)s->E * 4);
  return bytes + 256;
}

size_t moe_forward_workspace_size(const moe_shape* s) {
  if (check_shape(s, true, true) != MOE_OK) return 0;
  moe_workspace_layout L;
  layout_of(*s, &L);
  return L.total;
}

moe_status moe_forward_workspace_layout(const moe_shape* s, moe_workspace_layout* L) {
  if (L == nullptr) return MOE_ERR_INVALID_ARG;
  const moe_status r = check_shape(s, true, true);
  if (r != MOE_OK) return r;
  layout_of(*s, L);
  return MOE_OK;
}

moe_status moe_route(const moe_shape* s, const void* x, const void* w_r, const float* bias,
                     const float* logits_in, float* logits_out, int32_t* topk_ids, float* topk_w,
                     moe_stream_t stream) {
  moe_status r = check_shape(s, logits_in == nullptr, false);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;  // nothing to read or write; pointers may be NULL
  if (topk_ids == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
  if (logits_in == nullptr && (x == nullptr || w_r == nullptr)) return MOE_ERR_INVALID_ARG;
  if (logits_in == nullptr && !aligned16(x)) return MOE_ERR_INVALID_ARG;
  if (logits_in == nullptr && route_tc_supported(*s) && aligned16(w_r))
    return launch_route_tc(*s, x, w_r, bias, logits_out, topk_ids, topk_w, (cudaStream_t)stream);
  return launch_route(*s, x, w_r, bias, logits_in, logits_out, topk_ids, topk_w,
                      (cudaStream_t)stream);
}

moe_status moe_permute(const moe_shape* s, const int32_t* topk_ids, int32_t* counts,
                       int32_t* offsets, int32_t* assign_to_perm, int32_t* perm_to_assign,
                       const void* x, void* x_perm, void* workspace, size_t ws_bytes,
                       moe_stream_t stream) {
  const bool gather = (x != nullptr && x_perm != nullptr);
  moe_status r = check_shape(s, gather, false);
  if (r != MOE_OK) return r;
  if (s->tile_round > 0) return MOE_ERR_UNSUPPORTED;  // rounding needs the router logits
  if (s->T == 0) {  // no assignments: only counts and offsets (all zero) are written
    if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * s->E, st) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (s->E + 1), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (topk_ids == nullptr || counts == nullptr || offsets == nullptr || assign_to_perm == nullptr ||
      perm_to_assign == nullptr)
    return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (gather && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  const size_t need = permute_scratch_bytes(*s);
  if (need > 0 && (workspace == nullptr || ws_bytes < need)) return MOE_ERR_WORKSPACE;
  return launch_permute(*s, topk_ids, counts, offsets, assign_to_perm, perm_to_assign, x, x_perm,
                        workspace, (cudaStream_t)stream);
}

moe_status moe_permute_static(const moe_shape* s, const int32_t* topk_ids, int32_t* counts,
                              int32_t* offsets, int32_t* assign_to_perm, int32_t* perm_to_assign,
                              const void* x, void* x_perm, moe_stream_t stream) {
  const bool gather = (x != nullptr && x_perm != nullptr);
  moe_status r = check_shape(s, gather, false);
  if (r != MOE_OK) return r;
  if (s->tile_round > 0) return MOE_ERR_UNSUPPORTED;  // rounding needs the router logits
  if (topk_ids == nullptr || counts == nullptr || offsets == nullptr || assign_to_perm == nullptr ||
      perm_to_assign == nullptr)
    return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (gather && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) {
    const cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * s->E, st) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (s->E + 1), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  return launch_permute_static(*s, topk_ids, counts, offsets, assign_to_perm, perm_to_assign, x,
                               x_perm, (cudaStream_t)stream);
}

moe_status moe_dispatch(const moe_shape* s, const void* x, const void* w_r, const float* bias,
                        const float* logits_in, float* logits_out, int32_t* topk_ids,
                        float* topk_w, int32_t* counts, int32_t* offsets,
                        int32_t* assign_to_perm, int32_t* perm_to_assign, void* x_perm,
                        void* workspace, size_t ws_bytes, moe_stream_t stream) {
  const bool gather = x_perm != nullptr;
  moe_status r = check_shape(s, logits_in == nullptr || gather, false);
  if (r != MOE_OK) return r;
  if (s->T == 0)
    return moe_permute(s, topk_ids, counts, offsets, assign_to_perm, perm_to_assign, nullptr,
                       nullptr, workspace, ws_bytes, stream);
  if (!topk_ids || !topk_w || !counts || !offsets || !assign_to_perm || !perm_to_assign)
    return MOE_ERR_INVALID_ARG;
  if (gather && (x == nullptr || !aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if (rounds_up(*s)) return MOE_ERR_UNSUPPORTED;  // added assignments: moe_forward only
  if (s->tile_round > 0) {  // route, then the rounded permutation on the logits it saw
    const float* lg = logits_in != nullptr ? logits_in : logits_out;
    if (lg == nullptr) return MOE_ERR_INVALID_ARG;  // rounding reads the logits
    const size_t sb = align256(permute_scratch_bytes(*s));
    const size_t need = sb + align256((size_t)s->T * s->K * 4) + align256((size_t)s->E * 4);
    if (workspace == nullptr || ws_bytes < need || ((uintptr_t)workspace & 255) != 0)
      return MOE_ERR_WORKSPACE;
    if ((r = moe_route(s, x, w_r, bias, logits_in, logits_out, topk_ids, topk_w, stream)) != MOE_OK)
      return r;
    uint8_t* ws = (uint8_t*)workspace;
    return launch_permute_rounded(*s, topk_ids, lg, counts, offsets, assign_to_perm,
                                  perm_to_assign, gather ? x : nullptr, x_perm, ws,
                                  (int32_t*)(ws + sb),
                                  (int32_t*)(ws + sb + align256((size_t)s->T * s->K * 4)),
                                  (cudaStream_t)stream);
  }
  // every argument is checked before the first launch
  const size_t need = permute_scratch_bytes(*s);
  if (need > 0 && (workspace == nullptr || ws_bytes < need)) return MOE_ERR_WORKSPACE;
  if ((r = moe_route(s, x, w_r, bias, logits_in, logits_out, topk_ids, topk_w, stream)) != MOE_OK)
    return r;
  return moe_permute(s, topk_ids, counts, offsets, assign_to_perm, perm_to_assign,
                     gather ? x : nullptr, x_perm, workspace, ws_bytes, stream);
}

moe_status moe_grouped_ffn(const moe_shape* s, const void* x, const int32_t* offsets,
                           const int32_t* perm_to_assign, const void* w_gate, const void* w_up,
                           const void* w_down, void* a_act, void* y_perm, moe_stream_t stream) {
  moe_status r = check_shape(s, true, true);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!x || !offsets || !perm_to_assign || !w_gate || !w_up || !w_down || !a_act || !y_perm)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      !aligned16(a_act) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  if (s->dtype == MOE_BF16)
    return launch_ffn_tc_mixed(*s, x, offsets, perm_to_assign, w_gate, w_up, w_down, a_act, y_perm,
                               gateup_mode(*s), use_pair_down(*s), nullptr, (cudaStream_t)stream);
  return launch_ffn_simt(*s, x, offsets, perm_to_assign, w_gate, w_up, w_down, a_act, y_perm,
                         (cudaStream_t)stream);
}

moe_status moe_combine(const moe_shape* s, const void* y_perm, const int32_t* assign_to_perm,
                       const float* topk_w, void* out, moe_stream_t stream) {
  moe_status r = check_shape(s, true, false);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!y_perm || !assign_to_perm || !topk_w || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  return launch_combine(*s, y_perm, assign_to_perm, topk_w, out, (cudaStream_t)stream);
}


moe_status moe_forward(const moe_shape* s, const void* x, const void* w_r, const float* bias,
                       const float* logits_in, const void* w_gate, const void* w_up,
                       const void* w_down, void* out, void* workspace, size_t ws_bytes,
                       moe_stream_t stream) {
  return forward_impl(s, x, w_r, bias, logits_in, w_gate, w_up, w_down, out, nullptr, workspace,
                      ws_bytes, stream);
}

moe_status moe_forward_h(const moe_shape* s, const void* x, const void* w_r, const float* bias,
                         const float* logits_in, const void* w_gate, const void* w_up,
                         const void* w_down, void* out, void* h, void* workspace,
                         size_t ws_bytes, moe_stream_t stream) {
  if (s != nullptr && s->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (h == nullptr || !aligned16(h)) return MOE_ERR_INVALID_ARG;
  return forward_impl(s, x, w_r, bias, logits_in, w_gate, w_up, w_down, out, h, workspace,
                      ws_bytes, stream);
}

size_t moe_backward_workspace_size(const moe_shape* s) {
  if (check_shape(s, true, true) != MOE_OK) return 0;
  return align256(backward_scratch_bytes(*s, true)) + 256;
}

moe_status moe_backward(const moe_shape* s, const void* d_out, const float* topk_w,
                        const int32_t* offsets, const int32_t* perm_to_assign,
                        const int32_t* assign_to_perm, const void* w_gate, const void* w_up,
                        const void* w_down, const void* h, void* d_h, float* d_w, void* d_x,
                        void* workspace, size_t ws_bytes, moe_stream_t stream) {
  moe_status r = check_shape(s, true, true);
  if (r != MOE_OK) return r;
  if (s->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (s->T == 0) return MOE_OK;
  if (!d_out || !topk_w || !offsets || !perm_to_assign || !assign_to_perm || !w_down || !h ||
      !d_h || !d_w)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(d_out) || !aligned16(w_down) || !aligned16(h) || !aligned16(d_h))
    return MOE_ERR_INVALID_ARG;
  if (d_x != nullptr && (!w_gate || !w_up || !aligned16(w_gate) || !aligned16(w_up) ||
                         !aligned16(d_x)))
    return MOE_ERR_INVALID_ARG;
  const size_t need = backward_scratch_bytes(*s, d_x != nullptr);
  if (workspace == nullptr || ws_bytes < need || ((uintptr_t)workspace & 255) != 0)
    return MOE_ERR_WORKSPACE;
  return launch_backward(*s, d_out, topk_w, offsets, perm_to_assign, assign_to_perm, w_gate,
                         w_up, w_down, h, d_h, d_w, d_x, workspace, (cudaStream_t)stream);
}

moe_status moe_backward_router(const moe_shape* s, const void* x, const void* w_r,
                               const float* logits, const int32_t* topk_ids, const float* topk_w,
                               const float* d_w, float* d_logits, float* d_w_r, float* d_bias,
                               void* d_x, moe_stream_t stream) {
  moe_status r = check_shape(s, true, false);
  if (r != MOE_OK) return r;
  if (s->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (s->T == 0) {  // nothing routed: the weight and bias gradients are zero
    if (d_w_r == nullptr) return MOE_ERR_INVALID_ARG;
    const cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(d_w_r, 0, sizeof(float) * (size_t)s->d * s->E, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (d_bias != nullptr && cudaMemsetAsync(d_bias, 0, sizeof(float) * s->E, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (!x || !w_r || !topk_ids || !topk_w || !d_w || !d_logits || !d_w_r) return MOE_ERR_INVALID_ARG;
  if (!s->renormalize && logits == nullptr) return MOE_ERR_INVALID_ARG;  // the plain softmax
  if (d_x != nullptr && !aligned16(d_x)) return MOE_ERR_INVALID_ARG;
  if (s->E > 16 && !aligned16(x)) return MOE_ERR_INVALID_ARG;  // 16-byte row loads of x
  return launch_router_backward(*s, x, w_r, logits, topk_ids, topk_w, d_w, d_logits, d_w_r,
                                d_bias, d_x, (cudaStream_t)stream);
}

moe_status moe_get_device_status(moe_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return MOE_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return MOE_ERR_CUDA;
  return (moe_status)v;
}

const char* moe_status_string(moe_status st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_INDEX: return "device index out of range";
  }
  return "unknown status";
}

moe_status moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return MOE_OK;
}

moe_status moe_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_recs) {
    cudaEventSynchronize(r.b);
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  return MOE_OK;
}

int moe_kernel_count(void) { return K_COUNT; }

const char* moe_kernel_name(int id) { return (id >= 0 && id < K_COUNT) ? kKernelNames[id] : ""; }

moe_status moe_profile_query(int id, int64_t* launches, double* total_ms) {
  if (id < 0 || id >= K_COUNT || launches == nullptr || total_ms == nullptr)
    return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int64_t n = 0;
  double ms = 0.0;
  for (auto& r : g_recs) {
    if (r.kid != id) continue;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return MOE_ERR_CUDA;
    float f = 0.f;
    if (cudaEventElapsedTime(&f, r.a, r.b) != cudaSuccess) return MOE_ERR_CUDA;
    ++n;
    ms += f;
  }
  *launches = n;
  *total_ms = ms;
  return MOE_OK;
}

int64_t moe_launch_count(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  return g_launches;
}

moe_status moe_selftest_timeout(uint64_t limit_ns, moe_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  return launch_selftest_timeout(limit_ns, (cudaStream_t)stream);
}

}  // extern "C"
