// plan.cu -- batch plan: group a mixed batch's rows by adapter.
//
// A batch arrives with an index vector (row -> adapter id), the input of the
// segmented gather-and-multiply of "Multi-LoRA Serving: Why 100 Adapters Fit on
// One GPU" (section "How does one batch run 30 different adapters at once?").
// The plan kernel turns it into segments (rows of one adapter, in ascending
// slot order, rows ascending inside a segment) and cuts segments into work
// items of at most kItemRows rows, so that a work item reads its adapter's
// weights once for all of its rows.  A plan depends only on the batch, so one
// plan serves every adapted matrix of a forward step.
//
// One CTA of 1024 threads builds a plan: a shared-memory histogram over slots,
// one block-wide scan that places segments and items, and a stable scatter of
// the rows by a single warp (match_any groups equal ids inside a 32-row chunk;
// chunks go in row order, which makes the grouping stable).
#include "internal.cuh"

namespace lora {

struct Quad {
  int a, b, c, d;
};

__device__ __forceinline__ Quad quad_add(Quad x, Quad y) { return {x.a + y.a, x.b + y.b, x.c + y.c, x.d + y.d}; }

__device__ __forceinline__ Quad warp_inclusive_scan(Quad v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    Quad u;
    u.a = __shfl_up_sync(0xffffffffu, v.a, o);
    u.b = __shfl_up_sync(0xffffffffu, v.b, o);
    u.c = __shfl_up_sync(0xffffffffu, v.c, o);
    u.d = __shfl_up_sync(0xffffffffu, v.d, o);
    if (lane >= o) v = quad_add(v, u);
  }
  return v;
}

// Exclusive scan over the 1024 threads of the block; *total gets the sum.
__device__ Quad block_exclusive_scan(Quad v, Quad *s_warp, Quad *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Quad inc = warp_inclusive_scan(v, lane);
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    Quad t = s_warp[lane];
    s_warp[lane] = warp_inclusive_scan(t, lane);
  }
  __syncthreads();
  Quad base = warp > 0 ? s_warp[warp - 1] : Quad{0, 0, 0, 0};
  *total = s_warp[31];
  Quad ex = {base.a + inc.a - v.a, base.b + inc.b - v.b, base.c + inc.c - v.c, base.d + inc.d - v.d};
  __syncthreads();
  return ex;
}

__global__ void __launch_bounds__(kPlanThreads) plan_ids_kernel(const int32_t *__restrict__ ids, int T,
                                                                 PoolView pool, PlanView plan, int *status) {
  extern __shared__ int s_cnt[];  // [n_slots]: row count, then scatter cursor
  __shared__ Quad s_warp[32];
  __shared__ int s_bad_id, s_bad_empty;
  const int tid = threadIdx.x;
  const int n_slots = pool.n_slots;
  if (tid == 0) {
    s_bad_id = 0;
    s_bad_empty = 0;
  }
  for (int s = tid; s < n_slots; s += kPlanThreads) s_cnt[s] = 0;
  griddep_wait();
  griddep_launch_dependents();  // the delta kernel may set up while the plan is built
  __syncthreads();

  // 1. histogram of valid ids
  for (int t = tid; t < T; t += kPlanThreads) {
    int id = ids[t];
    if (id == -1) continue;
    if (id < -1 || id >= n_slots) {
      s_bad_id = 1;
      continue;
    }
    if (!pool.loaded[id]) {
      s_bad_empty = 1;
      continue;
    }
    atomicAdd(&s_cnt[id], 1);
  }
  __syncthreads();

  // 2. scan over slots: row offset, segment index, first item index
  Quad carry = {0, 0, 0, 0};
  for (int base = 0; base < n_slots; base += kPlanThreads) {
    const int s = base + tid;
    const int c = s < n_slots ? s_cnt[s] : 0;
    Quad v = {c, c > 0 ? 1 : 0, (c + kItemRows - 1) / kItemRows, 0};
    Quad tot;
    Quad ex = block_exclusive_scan(v, s_warp, &tot);
    if (c > 0) {
      const int off = carry.a + ex.a, seg = carry.b + ex.b, it = carry.c + ex.c;
      plan.seg_start[seg] = off;
      plan.seg_slot[seg] = s;
      plan.seg_row[seg] = -1;
      for (int k = 0; k * kItemRows < c; ++k)
        plan.items[it + k] = make_int4(s, off + k * kItemRows, min(kItemRows, c - k * kItemRows), seg);
      s_cnt[s] = off;  // becomes the cursor of the scatter
    }
    carry = quad_add(carry, tot);
  }
  if (tid == 0) {
    plan.seg_start[carry.b] = carry.a;
    plan.hdr[kHdrSegs] = carry.b;
    plan.hdr[kHdrActive] = carry.a;
    plan.hdr[kHdrItems] = carry.c;
    plan.hdr[kHdrTiles] = 0;
    plan.hdr[kHdrT] = T;
    plan.hdr[kHdrItemsAll] = carry.c;
  }
  __syncthreads();

  // 3. stable scatter of the rows, 32 rows at a time in row order
  if (tid < 32) {
    const unsigned lt = (1u << tid) - 1u;
    for (int base = 0; base < T; base += 32) {
      const int t = base + tid;
      const int id = t < T ? ids[t] : -1;
      const bool valid = t < T && id >= 0 && id < n_slots && pool.loaded[id];
      const int key = valid ? id : -2 - tid;  // invalid lanes never match anyone
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      const int leader = __ffs(peers) - 1;
      int pos = 0;
      if (valid && tid == leader) {
        pos = s_cnt[id];
        s_cnt[id] = pos + __popc(peers);
      }
      pos = __shfl_sync(0xffffffffu, pos, leader);
      if (valid) plan.perm[pos + __popc(peers & lt)] = t;
      __syncwarp();
    }
  }
  if (tid == 0) {
    if (s_bad_id) set_status(status, LORA_ERR_BAD_ID);
    else if (s_bad_empty) set_status(status, LORA_ERR_NOT_LOADED);
  }
}

// One pass over the segments (one per thread, S <= kPlanThreads): offsets,
// slot and validity are read together; a block scan places segments, decode
// items and tensor-core tiles; the decode items of the long segments (for
// targets the tensor cores cannot serve) and the row order are written from
// shared-memory copies of the segment table.  Larger S take the same steps
// in chunks of kPlanThreads segments, reading the table back from the plan.
__global__ void __launch_bounds__(kPlanThreads) plan_segments_kernel(const int32_t *__restrict__ seg_off,
                                                                      const int32_t *__restrict__ seg_slot,
                                                                      int S, int T, int mma_min, PoolView pool,
                                                                      PlanView plan, int *status) {
  __shared__ Quad s_warp[32];
  __shared__ int s_bad_id, s_bad_empty;
  __shared__ int s_start[kPlanThreads + 1], s_row[kPlanThreads];
  const int tid = threadIdx.x;
  const bool one_pass = S <= kPlanThreads;
  if (tid == 0) {
    s_bad_id = 0;
    s_bad_empty = 0;
  }
  griddep_wait();
  griddep_launch_dependents();
  // Offsets must be non-decreasing and inside [0, T] (then segments are
  // disjoint); otherwise the whole plan is empty.  (In one pass the slot and
  // its loaded flag are read at the same time.)
  int b0 = 0, e0 = 0, slot0 = -1, loaded0 = 0;
  bool malformed = false;
  for (int s = tid; s < S; s += kPlanThreads) {
    const int b = seg_off[s], e = seg_off[s + 1];
    if (b < 0 || e < b || e > T) malformed = true;
    if (one_pass) {
      b0 = b;
      e0 = e;
      slot0 = seg_slot[s];
      if (slot0 >= 0 && slot0 < pool.n_slots) loaded0 = pool.loaded[slot0];
    }
  }
  if (__syncthreads_or(malformed)) {
    if (tid == 0) {
      plan.seg_start[0] = 0;
      plan.hdr[kHdrSegs] = 0;
      plan.hdr[kHdrActive] = 0;
      plan.hdr[kHdrItems] = 0;
      plan.hdr[kHdrTiles] = 0;
      plan.hdr[kHdrT] = T;
      plan.hdr[kHdrItemsAll] = 0;
      set_status(status, LORA_ERR_BAD_ID);
    }
    return;
  }
  Quad carry = {0, 0, 0, 0};
  for (int base = 0; base < S; base += kPlanThreads) {
    const int s = base + tid;
    int b = 0, len = 0, slot = -1;
    if (s < S) {
      int e, ld;
      if (one_pass) {
        b = b0;
        e = e0;
        slot = slot0;
        ld = loaded0;
      } else {
        b = seg_off[s];
        e = seg_off[s + 1];
        slot = seg_slot[s];
        ld = (slot >= 0 && slot < pool.n_slots) ? pool.loaded[slot] : 0;
      }
      if (slot == -1 || e == b) {
        // no adapter, or an empty segment: nothing to do
      } else if (slot < -1 || slot >= pool.n_slots) {
        s_bad_id = 1;
      } else if (!ld) {
        s_bad_empty = 1;
      } else {
        len = e - b;
      }
    }
    const bool mma = len >= mma_min;
    // c: decode items of short segments; d: tiles of long segments
    Quad v = {len, len > 0 ? 1 : 0, (len > 0 && !mma) ? (len + kItemRows - 1) / kItemRows : 0,
              mma ? (len + kMmaRows - 1) / kMmaRows : 0};
    Quad tot;
    Quad ex = block_exclusive_scan(v, s_warp, &tot);
    if (len > 0) {
      const int off = carry.a + ex.a, seg = carry.b + ex.b;
      plan.seg_start[seg] = off;
      plan.seg_slot[seg] = slot;
      plan.seg_row[seg] = b;
      if (one_pass) {
        s_start[seg] = off;
        s_row[seg] = b;
      }
      if (mma) {
        const int j0 = carry.d + ex.d;
        for (int k = 0; k * kMmaRows < len; ++k) {
          const int m = min(kMmaRows, len - k * kMmaRows);
          plan.tiles[j0 + k] = make_int4(slot, b + k * kMmaRows, m, seg);
          if (one_pass)  // its decode items, after all the short segments' ones
            for (int q = 0; q < kMmaRows / kItemRows; ++q)
              plan.items[tot.c + (j0 + k) * (kMmaRows / kItemRows) + q] =
                  make_int4(slot, off + k * kMmaRows + q * kItemRows, max(0, min(kItemRows, m - q * kItemRows)), seg);
        }
      } else {
        const int i0 = carry.c + ex.c;
        for (int k = 0; k * kItemRows < len; ++k)
          plan.items[i0 + k] = make_int4(slot, off + k * kItemRows, min(kItemRows, len - k * kItemRows), seg);
      }
    }
    carry = quad_add(carry, tot);
  }
  const int n_tiles = carry.d, n_short = carry.c;
  if (!one_pass) {
    // Decode items for the long segments too (after the short ones).  Each
    // tile of kMmaRows rows becomes kMmaRows / kItemRows items.
    __syncthreads();
    for (int idx = tid; idx < n_tiles * (kMmaRows / kItemRows); idx += kPlanThreads) {
      const int j = idx / (kMmaRows / kItemRows), q = idx - j * (kMmaRows / kItemRows);
      const int4 t = plan.tiles[j];
      const int first = t.y - plan.seg_row[t.w] + plan.seg_start[t.w] + q * kItemRows;  // perm index
      const int m = min(kItemRows, t.z - q * kItemRows);
      plan.items[n_short + idx] = m > 0 ? make_int4(t.x, first, m, t.w) : make_int4(t.x, first, 0, t.w);
    }
  }
  if (tid == 0) {
    plan.seg_start[carry.b] = carry.a;
    if (one_pass) s_start[carry.b] = carry.a;
    plan.hdr[kHdrSegs] = carry.b;
    plan.hdr[kHdrActive] = carry.a;
    plan.hdr[kHdrItems] = carry.c;
    plan.hdr[kHdrTiles] = carry.d;
    plan.hdr[kHdrT] = T;
    plan.hdr[kHdrItemsAll] = n_short + n_tiles * (kMmaRows / kItemRows);
  }
  __syncthreads();
  // perm: the rows of segment g are seg_row[g] .. seg_row[g] + length - 1
  const int n_segs = carry.b, n_active = carry.a;
  const int *starts = one_pass ? s_start : plan.seg_start;
  const int *rows = one_pass ? s_row : plan.seg_row;
  for (int p = tid; p < n_active; p += kPlanThreads) {
    int lo = 0, hi = n_segs - 1;
    while (lo < hi) {  // last segment whose start is <= p
      const int mid = (lo + hi + 1) >> 1;
      if (starts[mid] <= p) lo = mid;
      else hi = mid - 1;
    }
    plan.perm[p] = rows[lo] + (p - starts[lo]);
  }
  if (tid == 0) {
    if (s_bad_id) set_status(status, LORA_ERR_BAD_ID);
    else if (s_bad_empty) set_status(status, LORA_ERR_NOT_LOADED);
  }
}

int launch_plan_ids(lora_pool *pool, const int32_t *ids, int T, void *ws, cudaStream_t st) {
  PlanLayout L = plan_layout(T);
  size_t smem = size_t(pool->n_slots) * 4;
  static bool attr_set[64] = {};
  if (pool->device < 64 && !attr_set[pool->device]) {
    if (cudaFuncSetAttribute(plan_ids_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSlots * 4) !=
        cudaSuccess)
      return LORA_ERR_CUDA;
    attr_set[pool->device] = true;
  }
  g_launches.fetch_add(1);
  plan_ids_kernel<<<1, kPlanThreads, smem, st>>>(ids, T, pool->view(), plan_view(ws, L), pool->d_status);
  return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

int launch_plan_segments(lora_pool *pool, const int32_t *off, const int32_t *slot, int S, int T, void *ws,
                         cudaStream_t st) {
  PlanLayout L = plan_layout(T);
  g_launches.fetch_add(1);
  plan_segments_kernel<<<1, kPlanThreads, 0, st>>>(off, slot, S, T, segment_mma_min(S, T), pool->view(), plan_view(ws, L),
                                                   pool->d_status);
  return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
}

}  // namespace lora
