// capi.cu -- the compute entry points of the C ABI: argument checks on the
// host, then the plan kernel and the delta kernels on the caller's stream.
// No call here allocates memory or synchronises the host.
#include <algorithm>

#include "internal.cuh"

using namespace lora;

namespace {

int check_call(const lora_pool *p, int target, int T, const void *ws, size_t ws_bytes) {
  if (!p) return LORA_ERR_INVALID_ARG;
  if (target < 0 || target >= p->n_targets) return LORA_ERR_INVALID_ARG;
  if (T < 0 || T > kMaxTokens) return LORA_ERR_INVALID_ARG;
  if (T == 0) return LORA_OK;
  if (!ws) return LORA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return LORA_ERR_ALIGNMENT;
  if (ws_bytes < plan_layout(T).total) return LORA_ERR_WORKSPACE;
  return LORA_OK;
}

int check_rows(const void *ptr, int ld, int width) {
  if (!ptr) return LORA_ERR_INVALID_ARG;
  if (ld < width) return LORA_ERR_INVALID_ARG;
  if (!aligned16(ptr) || (ld % 8) != 0) return LORA_ERR_ALIGNMENT;
  return LORA_OK;
}

// x and y must not overlap (x is read while y is written).
bool overlap(const void *x, int ldx, const void *y, int ldy, int T) {
  const char *xa = static_cast<const char *>(x), *ya = static_cast<const char *>(y);
  const char *xb = xa + size_t(T) * ldx * 2, *yb = ya + size_t(T) * ldy * 2;
  return xa < yb && ya < xb;
}

// Operands of the fused layer: x [T, d_in], W [d_out, d_in], y [T, d_out];
// y overlaps neither x nor W.
int check_linear(const lora_pool *p, int target, const void *x, int ldx, const void *W, int ldw, const void *y,
                 int ldy, const int32_t *ids, const float *scales, int T) {
  const int d_in = p->targets[target].d_in, d_out = p->targets[target].d_out;
  int rc;
  if ((rc = check_rows(x, ldx, d_in)) != LORA_OK) return rc;
  if ((rc = check_rows(y, ldy, d_out)) != LORA_OK) return rc;
  if ((rc = check_rows(W, ldw, d_in)) != LORA_OK) return rc;
  if (!ids || !scales) return LORA_ERR_INVALID_ARG;
  if (overlap(x, ldx, y, ldy, T)) return LORA_ERR_INVALID_ARG;
  const char *wa = static_cast<const char *>(W), *ya = static_cast<const char *>(y);
  if (wa < ya + size_t(T) * ldy * 2 && ya < wa + size_t(d_out) * ldw * 2) return LORA_ERR_INVALID_ARG;
  return LORA_OK;
}

// kPlanSegmentsTiles: a segment plan that sent every segment to the
// tensor-core tiles (segment_mma_min == 1): no short-segment decode items.
enum { kPlanUnknown = 0, kPlanIds = 1, kPlanSegments = 2, kPlanSegmentsTiles = 3 };

void set_plan_kind(lora_pool *p, const void *ws, int kind) {
  std::lock_guard<std::mutex> lk(p->mu);
  p->plan_kind[ws] = kind;
}

int plan_kind(lora_pool *p, const void *ws) {
  std::lock_guard<std::mutex> lk(p->mu);
  auto it = p->plan_kind.find(ws);
  return it == p->plan_kind.end() ? kPlanUnknown : it->second;
}

}  // namespace

extern "C" {

size_t lora_workspace_bytes(const lora_pool *p, int target, int max_tokens) {
  if (!p || target < 0 || target >= p->n_targets || max_tokens < 0 || max_tokens > kMaxTokens) return 0;
  const size_t plan = plan_layout(max_tokens).total;
  const size_t scratch = prefill_scratch_bytes(p, target, max_tokens);
  return scratch ? align256(plan) + scratch : plan;
}

int lora_plan_layout_get(const lora_pool *p, int T, lora_plan_layout *out) {
  if (!p || !out || T < 0 || T > kMaxTokens) return LORA_ERR_INVALID_ARG;
  PlanLayout L = plan_layout(T);
  out->header = L.header;
  out->perm = L.perm;
  out->seg_start = L.seg_start;
  out->seg_slot = L.seg_slot;
  out->items = L.items;
  out->tiles = L.tiles;
  out->total = L.total;
  out->s_max = L.s_max;
  out->i_max = L.i_max;
  out->j_max = L.j_max;
  return LORA_OK;
}

int lora_mma_min_rows(void) { return kMmaMinRows; }

int lora_mma_min_rows_for(int S, int T) {
  if (S < 0 || T < 0 || T > kMaxTokens) return -1;
  return segment_mma_min(S, T);
}

void lora_set_wait_limit_ns(uint64_t ns) { set_wait_limit_ns(ns); }

int lora_plan_ids(lora_pool *p, const int32_t *ids, int T, void *ws, size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_plan_ids");
  int rc = check_call(p, 0, T, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  if (!ids) return LORA_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  rc = launch_plan_ids(p, ids, T, ws, static_cast<cudaStream_t>(stream));
  if (rc == LORA_OK) set_plan_kind(p, ws, kPlanIds);
  return rc;
}

int lora_plan_segments(lora_pool *p, const int32_t *seg_offsets, const int32_t *seg_slot, int S, int T, void *ws,
                       size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_plan_segments");
  int rc = check_call(p, 0, T, ws, ws_bytes);
  if (rc != LORA_OK) return rc;
  if (S < 0 || S > kMaxTokens) return LORA_ERR_INVALID_ARG;
  if (T == 0) return LORA_OK;
  if (S > 0 && (!seg_offsets || !seg_slot)) return LORA_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  rc = launch_plan_segments(p, seg_offsets, seg_slot, S, T, ws, static_cast<cudaStream_t>(stream));
  if (rc == LORA_OK) set_plan_kind(p, ws, segment_mma_min(S, T) == 1 ? kPlanSegmentsTiles : kPlanSegments);
  return rc;
}

int lora_apply_plan(lora_pool *p, int target, const void *x, int ldx, void *y, int ldy, const float *scales, int T,
                    const void *ws, size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_apply_plan");
  int rc = check_call(p, target, T, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  if ((rc = check_rows(x, ldx, p->targets[target].d_in)) != LORA_OK) return rc;
  if ((rc = check_rows(y, ldy, p->targets[target].d_out)) != LORA_OK) return rc;
  if (!scales) return LORA_ERR_INVALID_ARG;
  if (overlap(x, ldx, y, ldy, T)) return LORA_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int kind = plan_kind(p, ws);
  DecodeCall c;
  c.targets = &target;
  c.x = x;
  c.ldx = ldx;
  c.y = y;
  c.ldy = ldy;
  c.scales = scales;
  c.T = T;
  c.ws = const_cast<void *>(ws);
  if (kind == kPlanIds)  // index-vector plans hold decode items only
    return launch_decode(p, c, st);
  PrefillGeometry geo;
  if (kind == kPlanSegmentsTiles && prefill_geometry(p, target, plan_layout(T).j_max, &geo))
    return launch_prefill(p, target, x, ldx, y, ldy, scales, T, ws, ws_bytes, st);  // every segment
  if (kind == kPlanSegments && prefill_geometry(p, target, plan_layout(T).j_max, &geo)) {
    // short segments on the decode kernel, long ones on the tensor cores
    rc = launch_decode(p, c, st);
    if (rc != LORA_OK) return rc;
    return launch_prefill(p, target, x, ldx, y, ldy, scales, T, ws, ws_bytes, st);
  }
  // every segment on the decode kernel
  c.items_hdr = kHdrItemsAll;
  return launch_decode(p, c, st);
}

int lora_apply(lora_pool *p, int target, const void *x, int ldx, void *y, int ldy, const int32_t *ids,
               const float *scales, int T, void *ws, size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_apply");
  int rc = check_call(p, target, T, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  if ((rc = check_rows(x, ldx, p->targets[target].d_in)) != LORA_OK) return rc;
  if ((rc = check_rows(y, ldy, p->targets[target].d_out)) != LORA_OK) return rc;
  if (!scales || !ids) return LORA_ERR_INVALID_ARG;
  if (overlap(x, ldx, y, ldy, T)) return LORA_ERR_INVALID_ARG;
  if (T <= kFusedMaxT) {  // one launch: the delta kernel groups the rows itself
    DeviceGuard g(p->device);
    DecodeCall c;
    c.targets = &target;
    c.x = x;
    c.ldx = ldx;
    c.y = y;
    c.ldy = ldy;
    c.scales = scales;
    c.T = T;
    c.ws = ws;
    c.ids = ids;
    return launch_decode(p, c, static_cast<cudaStream_t>(stream));
  }
  if ((rc = lora_plan_ids(p, ids, T, ws, ws_bytes, stream)) != LORA_OK) return rc;
  return lora_apply_plan(p, target, x, ldx, y, ldy, scales, T, ws, ws_bytes, stream);
}

int lora_selftest_stalled_apply(lora_pool *p, int target, const void *x, int ldx, void *y, int ldy,
                                const int32_t *ids, const float *scales, int T, void *stream) {
  NvtxRange nvtx_range("lora_selftest_stalled_apply");
  if (!p || target < 0 || target >= p->n_targets || T < 0 || T > kFusedMaxT) return LORA_ERR_INVALID_ARG;
  if (T == 0) return LORA_OK;
  int rc;
  if ((rc = check_rows(x, ldx, p->targets[target].d_in)) != LORA_OK) return rc;
  if ((rc = check_rows(y, ldy, p->targets[target].d_out)) != LORA_OK) return rc;
  if (!scales || !ids) return LORA_ERR_INVALID_ARG;
  if (overlap(x, ldx, y, ldy, T)) return LORA_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  DecodeCall c;
  c.targets = &target;
  c.x = x;
  c.ldx = ldx;
  c.y = y;
  c.ldy = ldy;
  c.scales = scales;
  c.T = T;
  c.ids = ids;
  c.stall = 1;
  return launch_decode(p, c, static_cast<cudaStream_t>(stream));
}

int lora_apply_multi(lora_pool *p, int n_targets, const int *targets, const void *x, int ldx, void *y, int ldy,
                     const int *y_cols, const int32_t *ids, const float *scales, int T, void *ws, size_t ws_bytes,
                     void *stream) {
  NvtxRange nvtx_range("lora_apply_multi");
  if (!p || !targets || !y_cols || n_targets < 1 || n_targets > kMaxMulti) return LORA_ERR_INVALID_ARG;
  int rc = check_call(p, targets[0], T, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  const int d_in = p->targets[targets[0]].d_in, d_out = p->targets[targets[0]].d_out;
  for (int i = 0; i < n_targets; ++i) {
    const int t = targets[i];
    if (t < 0 || t >= p->n_targets) return LORA_ERR_INVALID_ARG;
    if (p->targets[t].d_in != d_in || p->targets[t].d_out != d_out) return LORA_ERR_INVALID_ARG;
    if (y_cols[i] < 0 || (long long)y_cols[i] + d_out > ldy) return LORA_ERR_INVALID_ARG;
    if (y_cols[i] % 8) return LORA_ERR_ALIGNMENT;
    for (int k = 0; k < i; ++k)  // the targets' column ranges must not overlap
      if (y_cols[k] < y_cols[i] + d_out && y_cols[i] < y_cols[k] + d_out) return LORA_ERR_INVALID_ARG;
  }
  if ((rc = check_rows(x, ldx, d_in)) != LORA_OK) return rc;
  if ((rc = check_rows(y, ldy, d_out)) != LORA_OK) return rc;
  if (!scales || !ids) return LORA_ERR_INVALID_ARG;
  if (overlap(x, ldx, y, ldy, T)) return LORA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DecodeCall c;
  c.n_tgt = n_targets;
  c.targets = targets;
  c.y_cols = y_cols;
  c.x = x;
  c.ldx = ldx;
  c.y = y;
  c.ldy = ldy;
  c.scales = scales;
  c.T = T;
  c.ws = ws;
  if (T <= kFusedMaxT) {
    DeviceGuard g(p->device);
    c.ids = ids;
    return launch_decode(p, c, st);
  }
  if ((rc = lora_plan_ids(p, ids, T, ws, ws_bytes, stream)) != LORA_OK) return rc;
  DeviceGuard g(p->device);
  return launch_decode(p, c, st);
}

int lora_apply_segments(lora_pool *p, int target, const void *x, int ldx, void *y, int ldy,
                        const int32_t *seg_offsets, const int32_t *seg_slot, int S, const float *scales, int T,
                        void *ws, size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_apply_segments");
  int rc = check_call(p, target, T, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  if ((rc = check_rows(x, ldx, p->targets[target].d_in)) != LORA_OK) return rc;
  if ((rc = check_rows(y, ldy, p->targets[target].d_out)) != LORA_OK) return rc;
  if (!scales) return LORA_ERR_INVALID_ARG;
  if (overlap(x, ldx, y, ldy, T)) return LORA_ERR_INVALID_ARG;
  if ((rc = lora_plan_segments(p, seg_offsets, seg_slot, S, T, ws, ws_bytes, stream)) != LORA_OK) return rc;
  return lora_apply_plan(p, target, x, ldx, y, ldy, scales, T, ws, ws_bytes, stream);
}

int lora_shrink(lora_pool *p, int target, const void *x, int ldx, const int32_t *ids, int T, float *v, int ldv,
                void *ws, size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_shrink");
  int rc = check_call(p, target, T, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  if ((rc = check_rows(x, ldx, p->targets[target].d_in)) != LORA_OK) return rc;
  if (!ids || !v || ldv < p->r_max) return LORA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(v) & 3u) return LORA_ERR_ALIGNMENT;
  DecodeCall c;
  c.mode = kShrinkOnly;
  c.targets = &target;
  c.x = x;
  c.ldx = ldx;
  c.v = v;
  c.ldv = ldv;
  c.T = T;
  c.ws = ws;
  if (T <= kFusedMaxT) {
    DeviceGuard g(p->device);
    c.ids = ids;
    return launch_decode(p, c, static_cast<cudaStream_t>(stream));
  }
  if ((rc = lora_plan_ids(p, ids, T, ws, ws_bytes, stream)) != LORA_OK) return rc;
  DeviceGuard g(p->device);
  return launch_decode(p, c, static_cast<cudaStream_t>(stream));
}

int lora_expand(lora_pool *p, int target, const float *v, int ldv, void *y, int ldy, const int32_t *ids,
                const float *scales, int T, void *ws, size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_expand");
  int rc = check_call(p, target, T, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  if ((rc = check_rows(y, ldy, p->targets[target].d_out)) != LORA_OK) return rc;
  if (!ids || !v || !scales || ldv < p->r_max) return LORA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(v) & 3u) return LORA_ERR_ALIGNMENT;
  DecodeCall c;
  c.mode = kExpandOnly;
  c.targets = &target;
  c.y = y;
  c.ldy = ldy;
  c.scales = scales;
  c.v = const_cast<float *>(v);
  c.ldv = ldv;
  c.T = T;
  c.ws = ws;
  if (T <= kFusedMaxT) {
    DeviceGuard g(p->device);
    c.ids = ids;
    return launch_decode(p, c, static_cast<cudaStream_t>(stream));
  }
  if ((rc = lora_plan_ids(p, ids, T, ws, ws_bytes, stream)) != LORA_OK) return rc;
  DeviceGuard g(p->device);
  return launch_decode(p, c, static_cast<cudaStream_t>(stream));
}

size_t lora_linear_workspace_bytes(const lora_pool *p, int target, int max_tokens) {
  if (!p || target < 0 || target >= p->n_targets || max_tokens < 0 || max_tokens > kMaxTokens) return 0;
  return align256(plan_layout(max_tokens).total) + align256(size_t(max_tokens) * p->r_max * 4);
}

int lora_linear(lora_pool *p, int target, const void *x, int ldx, const void *W, int ldw, void *y, int ldy,
                const int32_t *ids, const float *scales, int T, void *ws, size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_linear");
  int rc = check_call(p, target, T, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  if ((rc = check_linear(p, target, x, ldx, W, ldw, y, ldy, ids, scales, T)) != LORA_OK) return rc;
  const size_t voff = align256(plan_layout(T).total);
  if (ws_bytes < voff + size_t(T) * p->r_max * 4) return LORA_ERR_WORKSPACE;
  float *v = reinterpret_cast<float *>(static_cast<char *>(ws) + voff);
  if ((rc = lora_shrink(p, target, x, ldx, ids, T, v, p->r_max, ws, ws_bytes, stream)) != LORA_OK) return rc;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  DeviceGuard g(p->device);
  return launch_linear(p, target, x, ldx, W, ldw, y, ldy, ids, scales, v, p->r_max, T, st);
}

int lora_linear_expand(lora_pool *p, int target, const void *x, int ldx, const void *W, int ldw, const float *v,
                       int ldv, void *y, int ldy, const int32_t *ids, const float *scales, int T, void *stream) {
  NvtxRange nvtx_range("lora_linear_expand");
  if (!p || target < 0 || target >= p->n_targets || T < 0 || T > kMaxTokens) return LORA_ERR_INVALID_ARG;
  if (T == 0) return LORA_OK;
  int rc = check_linear(p, target, x, ldx, W, ldw, y, ldy, ids, scales, T);
  if (rc != LORA_OK) return rc;
  if (!v || ldv < p->r_max) return LORA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(v) & 3u) return LORA_ERR_ALIGNMENT;
  DeviceGuard g(p->device);
  return launch_linear(p, target, x, ldx, W, ldw, y, ldy, ids, scales, v, ldv, T, static_cast<cudaStream_t>(stream));
}

size_t lora_moe_workspace_bytes(const lora_pool *p, int target, int max_pairs) {
  if (!p || target < 0 || target >= p->n_targets || max_pairs < 0 || max_pairs > kMaxTokens) return 0;
  return align256(plan_layout(max_pairs).total) + align256(size_t(max_pairs) * 4);
}

int lora_apply_moe(lora_pool *p, int target, const void *x, int ldx, void *y, int ldy, const int32_t *lora_ids,
                   const int32_t *topk_ids, int T, int top_k, int n_experts, const float *scales, void *ws,
                   size_t ws_bytes, void *stream) {
  NvtxRange nvtx_range("lora_apply_moe");
  if (!p || target < 0 || target >= p->n_targets || T < 0) return LORA_ERR_INVALID_ARG;
  if (top_k < 1 || n_experts < 1 || (long long)T * top_k > kMaxTokens) return LORA_ERR_INVALID_ARG;
  const int n_pairs = T * top_k;
  int rc = check_call(p, target, n_pairs, ws, ws_bytes);
  if (rc != LORA_OK || T == 0) return rc;
  if ((rc = check_rows(x, ldx, p->targets[target].d_in)) != LORA_OK) return rc;
  if ((rc = check_rows(y, ldy, p->targets[target].d_out)) != LORA_OK) return rc;
  if (!lora_ids || !topk_ids || !scales) return LORA_ERR_INVALID_ARG;
  {
    const char *xa = static_cast<const char *>(x), *ya = static_cast<const char *>(y);
    if (xa < ya + size_t(n_pairs) * ldy * 2 && ya < xa + size_t(T) * ldx * 2) return LORA_ERR_INVALID_ARG;
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  DecodeCall c;
  c.targets = &target;
  c.x = x;
  c.ldx = ldx;
  c.y = y;
  c.ldy = ldy;
  c.scales = scales;
  c.T = n_pairs;
  c.ws = ws;
  c.x_div = top_k;
  if (n_pairs <= kFusedMaxT) {  // pairs grouped inside the kernel from the routing itself
    DeviceGuard g(p->device);
    c.ids = lora_ids;
    c.moe_topk = topk_ids;
    c.moe_k = top_k;
    c.moe_e = n_experts;
    return launch_decode(p, c, st);
  }
  const size_t poff = align256(plan_layout(n_pairs).total);
  if (ws_bytes < poff + size_t(n_pairs) * 4) return LORA_ERR_WORKSPACE;
  int32_t *pair_ids = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + poff);
  {
    DeviceGuard g(p->device);
    if ((rc = launch_moe_pair_ids(p, lora_ids, topk_ids, n_pairs, top_k, n_experts, pair_ids, st)) != LORA_OK)
      return rc;
  }
  if ((rc = lora_plan_ids(p, pair_ids, n_pairs, ws, ws_bytes, stream)) != LORA_OK) return rc;
  DeviceGuard g(p->device);
  return launch_decode(p, c, st);  // the pairs' slots were planned into ws
}

}  // extern "C"
