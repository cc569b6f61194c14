// sgmv.cu -- decode path of the multi-LoRA delta: one launch for every adapter
// of a batch.
//
// For each work item (up to kItemRows rows that share adapter a) the kernel
// computes, per row t,
//     v = A_a x[t]                 (shrink: r_a dot products of length d_in)
//     y[t] += (alpha_a / r_a) B_a v (expand, fused with the scale and the
//                                   in-place accumulate)
// which is the per-request term of y = xW + (x A_i) B_i (alpha / r) on
// "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU" (section "Why can't you
// just merge LoRA weights into the base model?").  The adapter's weights are
// read from HBM once per work item, for all of its rows: the cost the same page
// attributes to multi-adapter batches is the adapter bytes (section "How does
// one batch run 30 different adapters at once?").
//
// B200 mapping.  A thread-block cluster of kClusterCtas CTAs owns one work
// item at a time.  CTA c of the cluster handles slice c of d_in for the shrink
// (split-K) and slice c of d_out for the expand.  Each CTA streams its slices
// of A / x and B^T / y through a kStages-deep shared-memory ring filled by 1-D
// bulk async copies (cp.async.bulk, no multicast) that complete on mbarriers;
// pool rows are located through the page table, piece by piece at page
// boundaries.  Shrink partial sums are reduced first across lanes by warp
// shuffles, then across the cluster through distributed shared memory in a
// fixed CTA order, so every CTA ends with the same fp32 v (deterministic, and
// independent of the other rows of the batch).  The expand then adds
// scale * (B v) to its y slice in fp32 and stores bf16 (round to nearest even).
#include <cooperative_groups.h>

#include <algorithm>

#include "internal.cuh"

namespace cg = cooperative_groups;

namespace lora {

struct DecodeArgs {
  PoolView pool;
  int target, d_in, d_out, r_max;
  long long a_off, bt_off;
  const uint16_t *x;
  long long ldx;
  uint16_t *y;
  long long ldy;
  const float *scales;
  const int32_t *hdr;
  const int32_t *perm;
  const int4 *items;
  float *v;
  long long ldv;
  int *status;
  int stage_bytes;
  int items_hdr;  // header word holding the item count to process
};

// Copy `bytes` of slot's logical range starting at `off` into dst, cut at
// page boundaries.  A missing page (slot unloaded under our feet) is replaced
// by page-free reads of the pool base and reported.
__device__ __forceinline__ void copy_pool_row(const PoolView &pool, int slot, long long off, uint32_t bytes,
                                              uint8_t *dst, uint64_t *bar, int *status) {
  while (bytes > 0) {
    long long room;
    const uint8_t *src = pool_addr(pool, slot, off, &room);
    uint32_t n = (uint32_t)min((long long)bytes, room);
    if (src == nullptr) {
      set_status(status, LORA_ERR_NOT_LOADED);
      src = pool.base;
    }
    bulk_g2s(dst, src, n, bar);
    dst += n;
    off += n;
    bytes -= n;
  }
}

// Reduce JB per-lane values over the 32 lanes of a warp.  After the call
// acc[0] of lane l holds the full sum of value index (l >> (5 - log2 JB)).
template <int JB>
__device__ __forceinline__ void warp_reduce_multi(float (&acc)[JB], int lane) {
  int off = 16;
#pragma unroll
  for (int n = JB; n > 1; n >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int q = 0; q < n / 2; ++q) {
      const float send = upper ? acc[q] : acc[q + n / 2];
      const float keep = upper ? acc[q + n / 2] : acc[q];
      acc[q] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
#pragma unroll
  for (; off >= 1; off >>= 1) acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], off);
}

template <int JB>
struct Log2 {
  static constexpr int v = JB == 1 ? 0 : JB == 2 ? 1 : JB == 4 ? 2 : 3;
};

// One shrink tile: columns [v_lo*8, v_lo*8 + wv*8) of the item's rows.  Warp w
// owns adapter rows j = w + 8q (q < JB); lane l owns the l-th 16-byte column
// vector.  Partial dot products accumulate into s_part[i][j] (this CTA's
// share of v), each (i, j) written by exactly one lane.
template <int JB>
__device__ __forceinline__ void shrink_tile(const uint8_t *buf, int act_base, int wv, int r, int m,
                                            float *s_part, int lane, int warp) {
  if (warp >= r) return;
  float a[JB][8];
#pragma unroll
  for (int q = 0; q < JB; ++q) {
    const int j = warp + 8 * q;
    if (j < r && lane < wv) {
      unpack8(*reinterpret_cast<const uint4 *>(buf + j * kTileRowBytes + lane * 16), a[q]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) a[q][e] = 0.f;
    }
  }
  const uint8_t *xb = buf + act_base;
  const int own_q = lane >> (5 - Log2<JB>::v);
  const bool writer = (lane & ((32 / JB) - 1)) == 0;
  for (int i = 0; i < m; ++i) {
    float xv[8];
    if (lane < wv) {
      unpack8(*reinterpret_cast<const uint4 *>(xb + i * kTileRowBytes + lane * 16), xv);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) xv[e] = 0.f;
    }
    float acc[JB];
#pragma unroll
    for (int q = 0; q < JB; ++q) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(a[q][e], xv[e], s);
      acc[q] = s;
    }
    warp_reduce_multi<JB>(acc, lane);
    const int j = warp + 8 * own_q;
    if (writer && j < r) s_part[i * kRMax + j] += acc[0];
  }
}

// One expand tile: columns [v_lo*8, v_lo*8 + wv*8) of d_out.  Warp w owns rows
// w and w + 8 of the item; lane l owns the l-th 16-byte column vector.
__device__ __forceinline__ void expand_tile(const uint8_t *buf, int act_base, int wv, int v_lo, int r, int m,
                                            const float *s_v, float scale, const int *s_rows,
                                            const DecodeArgs &a, int lane, int warp) {
  if (warp >= m || lane >= wv) return;
  const bool two = warp + 8 < m;
  float acc0[8], acc1[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    acc0[e] = 0.f;
    acc1[e] = 0.f;
  }
  const float *v0 = s_v + warp * kRMax;
  const float *v1 = s_v + (warp + 8) * kRMax;
  for (int j = 0; j < r; ++j) {
    float b[8];
    unpack8(*reinterpret_cast<const uint4 *>(buf + j * kTileRowBytes + lane * 16), b);
    const float c0 = v0[j];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc0[e] = fmaf(c0, b[e], acc0[e]);
    if (two) {
      const float c1 = v1[j];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc1[e] = fmaf(c1, b[e], acc1[e]);
    }
  }
  const uint8_t *yb = buf + act_base;
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    if (rr == 1 && !two) break;
    const int i = warp + 8 * rr;
    float yv[8];
    unpack8(*reinterpret_cast<const uint4 *>(yb + i * kTileRowBytes + lane * 16), yv);
    const float *acc = rr ? acc1 : acc0;
    uint4 o;
    o.x = pack_bf16x2(fmaf(scale, acc[0], yv[0]), fmaf(scale, acc[1], yv[1]));
    o.y = pack_bf16x2(fmaf(scale, acc[2], yv[2]), fmaf(scale, acc[3], yv[3]));
    o.z = pack_bf16x2(fmaf(scale, acc[4], yv[4]), fmaf(scale, acc[5], yv[5]));
    o.w = pack_bf16x2(fmaf(scale, acc[6], yv[6]), fmaf(scale, acc[7], yv[7]));
    const long long row = s_rows[i];
    *reinterpret_cast<uint4 *>(a.y + row * a.ldy + (long long)(v_lo + lane) * 8) = o;
  }
}

template <int MODE>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const DecodeArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int cid = blockIdx.x / C;
  const int ncl = gridDim.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *ring = smem;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * a.stage_bytes);
  float *s_part = reinterpret_cast<float *>(full + kStages);
  float *s_v = s_part + kItemRows * kRMax;
  int *s_rows = reinterpret_cast<int *>(s_v + kItemRows * kRMax);
  const int act_base = a.r_max * kTileRowBytes;  // activation rows follow r_max weight rows

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();

  const int n_items = a.hdr[a.items_hdr];
  const int nvi = a.d_in / 8, nvo = a.d_out / 8;
  const int per_i = (nvi + C - 1) / C, per_o = (nvo + C - 1) / C;
  const int kv0 = min(crank * per_i, nvi), kv1 = min(kv0 + per_i, nvi);
  const int nv0 = min(crank * per_o, nvo), nv1 = min(nv0 + per_o, nvo);
  const int nk = (MODE == kExpandOnly) ? 0 : (per_i + kTileVecs - 1) / kTileVecs;
  const int nn = (MODE == kShrinkOnly) ? 0 : (per_o + kTileVecs - 1) / kTileVecs;
  const int tpi = nk + nn;
  const int my_items = cid < n_items ? (n_items - cid + ncl - 1) / ncl : 0;
  const long long total_tiles = (long long)my_items * tpi;

  // Producer: warp 0 fills ring stage g % kStages with tile g.
  auto issue = [&](long long g) {
    const int li = (int)(g / tpi), tt = (int)(g % tpi);
    const int4 d = a.items[cid + li * ncl];
    const int slot = d.x, pbeg = d.y, m = d.z;
    const int r = a.pool.rank[slot * a.pool.n_targets + a.target];
    const int stage = (int)(g % kStages);
    uint8_t *buf = ring + stage * a.stage_bytes;
    const bool shrink = tt < nk;
    const int t_idx = shrink ? tt : tt - nk;
    const int v_lo = (shrink ? kv0 : nv0) + t_idx * kTileVecs;
    const int wv = max(0, min(v_lo + kTileVecs, shrink ? kv1 : nv1) - v_lo);
    const int rows = (wv > 0 && r > 0 && m > 0) ? r + m : 0;
    const uint32_t row_bytes = (uint32_t)wv * 16u;
    if (lane == 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)rows * row_bytes);
    __syncwarp();
    for (int idx = lane; idx < rows; idx += 32) {
      if (idx < r) {
        const long long off = shrink ? a.a_off + ((long long)idx * a.d_in + (long long)v_lo * 8) * 2
                                     : a.bt_off + ((long long)idx * a.d_out + (long long)v_lo * 8) * 2;
        copy_pool_row(a.pool, slot, off, row_bytes, buf + idx * kTileRowBytes, &full[stage], a.status);
      } else {
        const int i = idx - r;
        const long long row = a.perm[pbeg + i];
        const uint16_t *src = shrink ? a.x + row * a.ldx + (long long)v_lo * 8
                                     : a.y + row * a.ldy + (long long)v_lo * 8;
        bulk_g2s(buf + act_base + i * kTileRowBytes, src, row_bytes, &full[stage]);
      }
    }
  };

  if (warp == 0) {
    for (long long g = 0; g < total_tiles && g < kStages; ++g) issue(g);
  }

  auto exchange = [&](int m, int r) {
    cluster.sync();  // every CTA's partial sums are complete
    for (int idx = tid; idx < m * r; idx += kDecodeThreads) {
      const int i = idx / r, j = idx - (idx / r) * r;
      float sum = 0.f;
      for (int c = 0; c < C; ++c) sum += cluster.map_shared_rank(s_part, c)[i * kRMax + j];
      s_v[i * kRMax + j] = sum;
    }
    cluster.sync();  // peers are done reading this CTA's partials
  };

  long long g = 0;
  for (int li = 0; li < my_items; ++li) {
    const int4 d = a.items[cid + li * ncl];
    const int slot = d.x, pbeg = d.y, m = d.z;
    const int r = a.pool.rank[slot * a.pool.n_targets + a.target];
    const float scale = a.scales[slot];
    __syncthreads();  // the previous item no longer uses s_rows / s_part / s_v
    if (tid < m) s_rows[tid] = a.perm[pbeg + tid];
    if (MODE != kExpandOnly) {
      for (int idx = tid; idx < kItemRows * kRMax; idx += kDecodeThreads) s_part[idx] = 0.f;
    } else {
      for (int idx = tid; idx < m * r; idx += kDecodeThreads) {
        const int i = idx / r, j = idx - (idx / r) * r;
        s_v[i * kRMax + j] = a.v[(long long)a.perm[pbeg + i] * a.ldv + j];
      }
    }
    __syncthreads();
    const int jb = r <= 8 ? 1 : r <= 16 ? 2 : r <= 32 ? 4 : 8;
    for (int tt = 0; tt < tpi; ++tt, ++g) {
      if (MODE == kFused && tt == nk && r > 0 && m > 0) exchange(m, r);
      const int stage = (int)(g % kStages);
      const uint32_t parity = (uint32_t)((g / kStages) & 1);
      const bool ok = mbar_wait_bounded(&full[stage], parity, a.status);
      if (ok && r > 0 && m > 0) {
        const uint8_t *buf = ring + stage * a.stage_bytes;
        const bool shrink = tt < nk;
        const int t_idx = shrink ? tt : tt - nk;
        const int v_lo = (shrink ? kv0 : nv0) + t_idx * kTileVecs;
        const int wv = max(0, min(v_lo + kTileVecs, shrink ? kv1 : nv1) - v_lo);
        if (wv > 0) {
          if (shrink) {
            switch (jb) {
              case 1: shrink_tile<1>(buf, act_base, wv, r, m, s_part, lane, warp); break;
              case 2: shrink_tile<2>(buf, act_base, wv, r, m, s_part, lane, warp); break;
              case 4: shrink_tile<4>(buf, act_base, wv, r, m, s_part, lane, warp); break;
              default: shrink_tile<8>(buf, act_base, wv, r, m, s_part, lane, warp); break;
            }
          } else {
            expand_tile(buf, act_base, wv, v_lo, r, m, s_v, scale, s_rows, a, lane, warp);
          }
        }
      }
      __syncthreads();  // stage consumed by every thread
      if (warp == 0 && g + kStages < total_tiles) issue(g + kStages);
    }
    if (MODE == kShrinkOnly && r > 0 && m > 0) {
      exchange(m, r);
      if (crank == 0) {
        for (int idx = tid; idx < m * a.r_max; idx += kDecodeThreads) {
          const int i = idx / a.r_max, j = idx - (idx / a.r_max) * a.r_max;
          a.v[(long long)s_rows[i] * a.ldv + j] = j < r ? s_v[i * kRMax + j] : 0.f;
        }
      }
    }
  }
  griddep_launch_dependents();
}

static int decode_smem_bytes(int r_max, int *stage_bytes) {
  *stage_bytes = (r_max + kItemRows) * kTileRowBytes;
  return kStages * *stage_bytes + kStages * 8 + 2 * kItemRows * kRMax * 4 + kItemRows * 4;
}

template <int MODE>
static cudaError_t launch_mode(const DecodeArgs &a, int n_clusters, int smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_clusters * kClusterCtas);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClusterCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<MODE>, a);
}

int decode_setup(lora_pool *pool) {
  int stage;
  const int smem = decode_smem_bytes(pool->r_max, &stage);
  pool->decode_smem = smem;
  // The attribute is per function: set it to what the largest rank needs, so
  // that pools of different r_max can coexist.
  const int smem_cap = decode_smem_bytes(kRMax, &stage);
  if (cudaFuncSetAttribute(decode_kernel<kFused>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_cap) !=
          cudaSuccess ||
      cudaFuncSetAttribute(decode_kernel<kShrinkOnly>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_cap) !=
          cudaSuccess ||
      cudaFuncSetAttribute(decode_kernel<kExpandOnly>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_cap) !=
          cudaSuccess)
    return LORA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kClusterCtas);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClusterCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<kFused>, &cfg) != cudaSuccess || n < 1) return LORA_ERR_CUDA;
  pool->decode_max_clusters = n;
  return LORA_OK;
}

int launch_decode(lora_pool *pool, int mode, int target, const void *x, int ldx, void *y, int ldy,
                  const float *scales, float *v, int ldv, int T, const void *ws, cudaStream_t st) {
  return launch_decode_items(pool, mode, target, x, ldx, y, ldy, scales, v, ldv, T, ws, st, kHdrItems);
}

int launch_decode_items(lora_pool *pool, int mode, int target, const void *x, int ldx, void *y, int ldy,
                        const float *scales, float *v, int ldv, int T, const void *ws, cudaStream_t st,
                        int items_hdr) {
  PlanLayout L = plan_layout(T);
  PlanView pv = plan_view(const_cast<void *>(ws), L);
  DecodeArgs a;
  a.pool = pool->view();
  a.target = target;
  a.d_in = pool->targets[target].d_in;
  a.d_out = pool->targets[target].d_out;
  a.r_max = pool->r_max;
  a.a_off = pool->a_off[target];
  a.bt_off = pool->bt_off[target];
  a.x = static_cast<const uint16_t *>(x);
  a.ldx = ldx;
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.scales = scales;
  a.hdr = pv.hdr;
  a.perm = pv.perm;
  a.items = pv.items;
  a.v = v;
  a.ldv = ldv;
  a.status = pool->d_status;
  a.items_hdr = items_hdr;
  int stage;
  const int smem = decode_smem_bytes(pool->r_max, &stage);
  a.stage_bytes = stage;
  // Items are bounded by min(T, n_slots) segments plus T / kItemRows chunk
  // splits; clusters loop over items, so the grid never exceeds what fits.
  const long long bound = (long long)std::min(T, pool->n_slots) + (T + kItemRows - 1) / kItemRows;
  int n_clusters = (int)std::min<long long>(bound, (long long)pool->decode_max_clusters);
  if (n_clusters < 1) n_clusters = 1;
  cudaError_t e;
  g_launches.fetch_add(1);
  if (mode == kFused) e = launch_mode<kFused>(a, n_clusters, smem, st);
  else if (mode == kShrinkOnly) e = launch_mode<kShrinkOnly>(a, n_clusters, smem, st);
  else e = launch_mode<kExpandOnly>(a, n_clusters, smem, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

}  // namespace lora
