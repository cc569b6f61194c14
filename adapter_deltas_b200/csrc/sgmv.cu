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
// B200 mapping.  A thread-block cluster of kClusterCtas CTAs (4 for batches
// with many more items than clusters) owns one work unit -- an item on one
// target -- at a time.  CTA c of the cluster handles slice c of d_in for the
// shrink (split-K) and slice c of d_out for the expand.  Each CTA streams its
// slices of A / x and B^T / y through a two-stage shared-memory ring filled
// by 1-D bulk async copies (cp.async.bulk, no multicast, one per row slice)
// that complete on mbarriers; pool rows are located through the page table
// (pieces at page boundaries).  The shrink and the expand run on warp-level
// bf16 MMA.  Shrink partial sums are reduced over the warps in shared memory,
// then across the cluster through distributed shared memory (st.async pushes)
// in a fixed CTA order, so every CTA ends with the same fp32 v (deterministic,
// and independent of the other rows of the batch).  The expand then adds
// scale * (B v) to its y slice in fp32 and stores bf16 (round to nearest even).
// Batches of up to kFusedMaxT rows are grouped by adapter inside the kernel.
#include <algorithm>
#include <climits>

#include "internal.cuh"

namespace lora {

struct DecodeArgs {
  PoolView pool;
  int d_in, d_out, r_max;
  // targets of this launch: all share x, d_in and d_out; work unit u is
  // (item u / n_tgt, target u % n_tgt); target i writes its delta into
  // columns y_col[i] .. y_col[i] + d_out - 1 of y
  int n_tgt;
  int tgt[kMaxMulti];
  long long a_off[kMaxMulti], bt_off[kMaxMulti], y_col[kMaxMulti];
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
  int n_stages;
  int tile_vecs;  // 16-byte vectors per staged row (64 or 32)
  int row_pitch;  // bytes between staged rows (tile_vecs * 16 + 16)
  int items_hdr;  // header word holding the item count to process
  int items_cap;  // entries the plan's items array has room for
  const int32_t *ids;  // non-null: group the rows of ids[0 .. T) inside the kernel (T <= kFusedMaxT)
  int T;
  int x_div;           // row t reads x row t / x_div (1; top_k for routed expert pairs)
  // routed expert pairs (moe_topk non-null, in-kernel grouping): row p is the
  // pair (token p / moe_k, its (p % moe_k)-th expert), ids[] holds each
  // token's adapter, and the pair's slot is adapter * moe_e + expert
  const int32_t *moe_topk;
  int moe_k, moe_e;
};

// ------------------------------------------------------------ warp MMA
// The decode contractions are tiny (an item has at most 16 rows and the rank
// is at most 64), so they run on warp-level mma.sync m16n8k16 (bf16 inputs,
// fp32 accumulators in registers), fed by ldmatrix from the staged rows:
// one instruction does 16 x 8 x 16 multiply-adds on bf16 operands as they are,
// where the same work on the FMA pipes needs a conversion per element.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shrink: this warp's share of V[i][j] = sum_k x[i][k] A[j][k] over the
// tile's columns, accumulated in acc[n-tile][4] (rows g, g + 8 and columns
// 2t, 2t + 1 of each 8-rank n-tile; g = lane / 4, t = lane % 4).  The warps
// split the tile's 16-column k-steps.  Rows i >= m and ranks j >= r read row 0
// of their operand instead: an output element depends only on its own row of
// each operand, so those lanes' results are simply never spilled.  An odd
// last vector (8 columns) zeroes both operands' upper k half.
template <int JB>
__device__ __forceinline__ void shrink_mma(uint32_t buf_u, uint32_t act_u, int pitch, int wv, int r, int m,
                                           float (&acc)[JB < 2 ? 2 : JB][4], int lane, int warp) {
  constexpr int NT = JB < 2 ? 2 : JB;  // 8-rank n-tiles (loaded two at a time)
  const int ksteps = (wv + 1) / 2;     // 16 columns = two 16-byte vectors
  const int xr = (lane & 7) + ((lane >> 3) & 1) * 8, xk = (lane >> 4) * 16;
  const uint32_t xrow = act_u + (xr < m ? xr : 0) * pitch + xk;
  uint32_t arow[NT / 2];
#pragma unroll
  for (int p = 0; p < NT / 2; ++p) {
    const int j = (lane & 7) + (lane >> 4) * 8 + 16 * p, ak = ((lane >> 3) & 1) * 16;
    arow[p] = buf_u + (j < r ? j : 0) * pitch + ak;
  }
  for (int ks = warp; ks < ksteps; ks += kConsumerWarps) {
    const bool half = 2 * ks + 1 >= wv;
    uint32_t a[4];
    ldsm_x4(xrow + ks * 32, a);
    if (half) a[2] = a[3] = 0u;
#pragma unroll
    for (int p = 0; p < NT / 2; ++p) {
      uint32_t b[4];
      ldsm_x4(arow[p] + ks * 32, b);
      if (half) b[1] = b[3] = 0u;
      mma_bf16_16816(acc[2 * p], a, b[0], b[1]);
      mma_bf16_16816(acc[2 * p + 1], a, b[2], b[3]);
    }
  }
}

// This warp's partial V of the item -> red[i * r + j] (rows < m, ranks < r).
template <int JB>
__device__ __forceinline__ void shrink_spill(const float (&acc)[JB < 2 ? 2 : JB][4], int r, int m, float *red,
                                             int lane) {
  constexpr int NT = JB < 2 ? 2 : JB;
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int i = g + (h >> 1) * 8, j = nt * 8 + 2 * t + (h & 1);
      if (i < m && j < r) red[i * r + j] = acc[nt][h];
    }
  }
}

// Expand: y[i][n] = bf16_rn(y + scale * sum_j V[i][j] B^T[j][n]) for the
// tile's columns.  V enters the MMA as two bf16 terms (hi + lo: about 16 bits
// of each fp32 value), built in registers once per item; B^T rows are loaded
// transposed by ldmatrix.  Warp w takes the 16-column groups w, w + 8, ...
template <int JB>
struct ExpandA {
  static constexpr int KS = JB < 2 ? 1 : JB / 2;  // 16-rank k-steps
  uint32_t hi[KS][4], lo[KS][4];
};

template <int JB>
__device__ __forceinline__ void expand_prepare(const float *s_v, int r, int m, ExpandA<JB> &A, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < ExpandA<JB>::KS; ++ks) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // a0: (g, 2t), a1: (g+8, 2t), a2: (g, 2t+8), a3: (g+8, 2t+8)
      const int i = g + (q & 1) * 8, j = 16 * ks + 2 * t + (q >> 1) * 8;
      const float v0 = (i < m && j < r) ? s_v[i * kRMax + j] : 0.f;
      const float v1 = (i < m && j + 1 < r) ? s_v[i * kRMax + j + 1] : 0.f;
      const uint32_t h = pack_bf16x2(v0, v1);
      A.hi[ks][q] = h;
      A.lo[ks][q] = pack_bf16x2(v0 - bf16_lo(h), v1 - bf16_hi(h));
    }
  }
}

template <int JB>
__device__ __forceinline__ void expand_group(uint32_t buf_u, const uint8_t *yb, uint32_t zero_u, int pitch, int wv,
                                             int v_lo, int r, int m, const ExpandA<JB> &A, float scale,
                                             const int *s_rows, long long ycol, const DecodeArgs &a, int lane,
                                             int cg) {
  const int g = lane >> 2, t = lane & 3;
  const int bj = (lane & 7) + ((lane >> 3) & 1) * 8, bn = (lane >> 4) * 16;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int ks = 0; ks < ExpandA<JB>::KS; ++ks) {
    // ranks j >= r read 16 zero bytes: their V is zero and stale weights
    // (possibly not finite) must not meet it
    const int j = 16 * ks + bj;
    uint32_t b[4];
    ldsm_x4_t(j < r ? buf_u + j * pitch + cg * 32 + bn : zero_u + bn, b);
    mma_bf16_16816(acc[0], A.hi[ks], b[0], b[1]);
    mma_bf16_16816(acc[1], A.hi[ks], b[2], b[3]);
    mma_bf16_16816(acc[0], A.lo[ks], b[0], b[1]);
    mma_bf16_16816(acc[1], A.lo[ks], b[2], b[3]);
  }
  const int n_nt = 2 * cg + 1 < wv ? 2 : 1;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    if (nt >= n_nt) break;
    const int col = cg * 16 + nt * 8 + 2 * t;  // within the tile
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int i = g + hr * 8;
      if (i < m) {
        const uint32_t yv = *reinterpret_cast<const uint32_t *>(yb + i * pitch + col * 2);
        const uint32_t o = pack_bf16x2(fmaf(scale, acc[nt][2 * hr], bf16_lo(yv)),
                                       fmaf(scale, acc[nt][2 * hr + 1], bf16_hi(yv)));
        *reinterpret_cast<uint32_t *>(a.y + (long long)s_rows[i] * a.ldy + ycol + (long long)v_lo * 8 + col) = o;
      }
    }
  }
}

// The warp takes the 16-column groups warp, warp + 8, ... two at a time
// (independent MMA chains side by side).
template <int JB>
__device__ __forceinline__ void expand_mma(uint32_t buf_u, const uint8_t *yb, uint32_t zero_u, int pitch, int wv,
                                           int v_lo, int r, int m, const ExpandA<JB> &A, float scale,
                                           const int *s_rows, long long ycol, const DecodeArgs &a, int lane,
                                           int warp) {
  const int groups = (wv + 1) / 2;  // 16-column groups (an odd last vector is half a group)
  for (int cg = warp; cg < groups; cg += 2 * kConsumerWarps) {
    expand_group<JB>(buf_u, yb, zero_u, pitch, wv, v_lo, r, m, A, scale, s_rows, ycol, a, lane, cg);
    if (cg + kConsumerWarps < groups)
      expand_group<JB>(buf_u, yb, zero_u, pitch, wv, v_lo, r, m, A, scale, s_rows, ycol, a, lane,
                       cg + kConsumerWarps);
  }
}

// ------------------------------------------------------------ cluster helpers
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ uint32_t mapa_u32(uint32_t addr, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(cta));
  return r;
}
// Asynchronous 4-byte store into a peer CTA's shared memory that signals the
// peer's mbarrier with its byte count on arrival.
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(remote_addr),
               "r"(__float_as_uint(v)), "r"(remote_bar)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (data written by peer CTAs).
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t *bar, uint32_t parity, int *status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 255u) == 255u && global_timer_ns() - t0 > kSpinNs) break;
  }
  atomicCAS(status, 0, LORA_ERR_TIMEOUT);
  return false;
}

// Per-item facts a warp needs while it consumes an item.  Every warp keeps
// its own copy (it resolved the item itself when it began copying it), so no
// warp waits on another to learn what it is computing.
struct ItemInfo {
  int m, r;
  float scale;
  int ycol;  // first column of the unit's target in y
  int rows[kItemRows];
};

struct DecodeSmem {
  uint8_t *ring;
  uint64_t *full, *empty, *recv_full;
  uint8_t *zero;   // 32 zero bytes: the expand's operand rows beyond the rank
  ItemInfo *info;  // [kConsumerWarps][kItemSlots]
  float *red;      // [kConsumerWarps][kItemRows * r_max]: the warps' shrink partials
  float *v, *recv;
  // in-kernel grouping of an index vector (kFusedMaxT rows)
  int *f_key, *f_perm, *f_warp, *f_items;
  int4 *f_info, *f_slot;
  // this cluster's items, resolved once (reuse the two int4 arrays above
  // once the grouping is done): (slot, first row, rows, rank) and
  // (A page, B^T page, scale bits, -)
  int4 *it_rec, *it_res;
};

constexpr int kFusedBytes = kFusedMaxT * (4 + 4 + 4 + 16 + 16) + 64;

__device__ __forceinline__ DecodeSmem decode_carve(uint8_t *smem, const DecodeArgs &a) {
  DecodeSmem S;
  uint8_t *p = smem;
  S.ring = p; p += a.n_stages * a.stage_bytes;
  S.full = reinterpret_cast<uint64_t *>(p); p += kMaxStages * 8;
  S.empty = reinterpret_cast<uint64_t *>(p); p += kMaxStages * 8;
  S.recv_full = reinterpret_cast<uint64_t *>(p); p += 2 * 8;
  S.zero = p; p += 32;
  S.info = reinterpret_cast<ItemInfo *>(p); p += kConsumerWarps * kItemSlots * sizeof(ItemInfo);
  S.red = reinterpret_cast<float *>(p); p += kConsumerWarps * kItemRows * a.r_max * 4;
  S.v = reinterpret_cast<float *>(p); p += kItemRows * kRMax * 4;
  S.recv = reinterpret_cast<float *>(p); p += 2 * kClusterCtas * kItemRows * a.r_max * 4;  // [2][C][kItemRows * r_max]
  S.f_info = reinterpret_cast<int4 *>(p); p += kFusedMaxT * 16;
  S.f_slot = reinterpret_cast<int4 *>(p); p += kFusedMaxT * 16;
  S.f_items = reinterpret_cast<int *>(p); p += kFusedMaxT * 4;
  S.f_key = reinterpret_cast<int *>(p); p += kFusedMaxT * 4;
  S.f_perm = reinterpret_cast<int *>(p); p += kFusedMaxT * 4;
  S.f_warp = reinterpret_cast<int *>(p);
  S.it_rec = S.f_info;
  S.it_res = S.f_slot;
  return S;
}

// Grouping of an index vector inside the kernel, for batches of at most
// kFusedMaxT rows (every CTA computes the same result): the rows of each
// slot in ascending row order, slots in ascending order, cut into items of
// at most kItemRows rows -- the plan kernel's items, in the same order, plus
// items for slots that hold no adapter (rank 0: they change no row; the
// resolve step reports them).  Row t's place is found by counting the rows
// with a smaller slot, or the same slot and a smaller index.  Each row's
// thread also loads what resolving its slot needs -- rank, scale and the
// physical pages of this CTA's A and B^T slices (-1 when the slices do not
// lie on one page) -- while the rows are being ranked; the first row of each
// item keeps them in S.f_slot.  Items are packed as slot | start << 14 |
// m << 22.  Returns the item count; *any_bad is set when some id lies
// outside [-1, n_slots).
struct SliceGeo {
  long long a_first, a_last, b_first, b_last;  // logical byte range of the slices (first < 0: none)
};

__device__ __forceinline__ int slice_page(const PoolView &p, int slot, long long first, long long last) {
  if (first < 0) return -1;
  const long long pf = p.log2_page < 0 ? 0 : first >> p.log2_page;
  const long long pl = p.log2_page < 0 ? 0 : last >> p.log2_page;
  return pf == pl ? __ldg(p.pt + (long long)slot * p.pps + pf) : -1;
}

// Slot of routed pair p: -1 for a token without adapter; an adapter id below
// -1, an expert outside [0, moe_e) or a slot past the pool gives n_slots
// (reported as a bad id).
__device__ __forceinline__ int moe_pair_slot(const DecodeArgs &a, int p) {
  const int lo = a.ids[p / a.moe_k];
  if (lo == -1) return -1;
  const int e = a.moe_topk[p];
  if (lo < -1 || e < 0 || e >= a.moe_e) return a.pool.n_slots;
  const long long s = (long long)lo * a.moe_e + e;
  return s < a.pool.n_slots ? (int)s : a.pool.n_slots;
}

__device__ int fused_plan(const DecodeArgs &a, const DecodeSmem &S, int tid, const SliceGeo &geo, int *any_bad) {
  const int T = a.T;
  int key = INT_MAX, bad = 0;
  int4 sinfo = make_int4(0, -1, -1, 0);
  if (tid < T) {
    const int id = a.moe_topk ? moe_pair_slot(a, tid) : a.ids[tid];
    if (id != -1) {
      if (id < -1 || id >= a.pool.n_slots) {
        bad = 1;
      } else {
        key = id;
        const PoolView &p = a.pool;
        sinfo.x = p.rank[(long long)id * p.n_targets + a.tgt[0]];
        sinfo.y = slice_page(p, id, geo.a_first, geo.a_last);
        sinfo.z = slice_page(p, id, geo.b_first, geo.b_last);
        sinfo.w = a.scales ? __float_as_int(a.scales[id]) : 0;
      }
    }
  }
  S.f_key[tid] = key;
  *any_bad = __syncthreads_or(bad);
  if (blockIdx.x == 0 && tid == 0 && *any_bad) set_status(a.status, LORA_ERR_BAD_ID);
  const bool valid = key != INT_MAX;
  int less = 0, same = 0, same_before = 0;
  if (valid) {
    const int4 *k4 = reinterpret_cast<const int4 *>(S.f_key);  // keys past T are INT_MAX
    for (int u4 = 0; u4 < (T + 3) / 4; ++u4) {
      const int4 k = k4[u4];
      const int u = 4 * u4;
      less += (k.x < key) + (k.y < key) + (k.z < key) + (k.w < key);
      same += (k.x == key) + (k.y == key) + (k.z == key) + (k.w == key);
      same_before += ((k.x == key) & (u < tid)) + ((k.y == key) & (u + 1 < tid)) + ((k.z == key) & (u + 2 < tid)) +
                     ((k.w == key) & (u + 3 < tid));
    }
  }
  const int n_valid = __syncthreads_count(valid);
  if (valid) {
    const int pos = less + same_before;
    S.f_perm[pos] = tid;
    S.f_info[pos] = make_int4(key, same_before, same, 0);
    if (same_before % kItemRows == 0) S.f_slot[pos] = sinfo;
  }
  __syncthreads();
  // item starts: sorted positions whose offset inside their segment is a
  // multiple of kItemRows; a block scan numbers them in position order
  const int4 inf = tid < n_valid ? S.f_info[tid] : make_int4(0, 1, 0, 0);
  const int flag = (tid < n_valid && inf.y % kItemRows == 0) ? 1 : 0;
  const int lane = tid & 31, warp = tid >> 5;
  int incl = flag;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) S.f_warp[warp] = incl;
  __syncthreads();
  int base = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kDecodeThreads / 32; ++w) {
    const int c = S.f_warp[w];
    base += w < warp ? c : 0;
    total += c;
  }
  if (flag) S.f_items[base + incl - 1] = inf.x | (tid << 14) | (min(kItemRows, inf.z - inf.y) << 22);
  __syncthreads();
  return total;
}

__device__ __forceinline__ int4 unpack_item(int v) {
  return make_int4(v & 0x3FFF, (v >> 14) & 0xFF, (v >> 22) & 0x1F, 0);
}

// Where a warp's next copies come from: the item it is copying, with the
// addresses of its rows held by the lanes (lane L: weight rows L and L + 32,
// activation row L).
struct IssueState {
  int li, tt;
  int slot, m, r;
  bool split_a, split_b;
  long long a_off, bt_off;  // the unit's target blocks inside a slot
  unsigned long long wa0, wa1, wb0, wb1, xrow, yrow;
};

template <int MODE, int JB>
__global__ void __launch_bounds__(kDecodeThreads, JB >= 8 ? 1 : 2) decode_kernel(const DecodeArgs a) {
  const int C = (int)cluster_nctarank();
  const int crank = (int)cluster_ctarank();
  const int cid = blockIdx.x / C, ncl = gridDim.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NS = a.n_stages;

  extern __shared__ __align__(128) uint8_t smem[];
  const DecodeSmem S = decode_carve(smem, a);
  ItemInfo *my_info = S.info + warp * kItemSlots;
  const int TV = a.tile_vecs, pitch = a.row_pitch;
  const int act_base = a.r_max * pitch;  // activation rows follow r_max weight rows
  const int recv_slice = kItemRows * a.r_max;    // floats one source CTA may send per item

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.full[s], kConsumerWarps);    // every warp announces its rows' bytes; the copies count them down
      mbar_init(&S.empty[s], kConsumerWarps);   // every warp arrives once it is done with the tile
    }
    mbar_init(&S.recv_full[0], 1);
    mbar_init(&S.recv_full[1], 1);
    fence_mbar_init();
  }
  if (tid < 8) reinterpret_cast<uint32_t *>(S.zero)[tid] = 0u;
  __syncthreads();
  // Peers may push into this CTA's shared memory only after its barriers are
  // initialised: arrive now, wait before the first push.
  cluster_arrive_relaxed();
  griddep_wait();
  griddep_launch_dependents();

  const int nvi = a.d_in / 8, nvo = a.d_out / 8;
  const int per_i = (nvi + C - 1) / C, per_o = (nvo + C - 1) / C;
  const int kv0 = min(crank * per_i, nvi), kv1 = min(kv0 + per_i, nvi);
  const int nv0 = min(crank * per_o, nvo), nv1 = min(nv0 + per_o, nvo);
  // logical byte ranges of this CTA's A and B^T slices of target i, rows
  // 0 .. r_max-1
  auto slice_geo = [&](int i) {
    SliceGeo g;
    g.a_first = g.b_first = -1;
    g.a_last = g.b_last = -1;
    if (MODE != kExpandOnly && kv1 > kv0) {
      g.a_first = a.a_off[i] + (long long)kv0 * 16;
      g.a_last = a.a_off[i] + ((long long)(a.r_max - 1) * a.d_in + (long long)kv1 * 8) * 2 - 1;
    }
    if (MODE != kShrinkOnly && nv1 > nv0) {
      g.b_first = a.bt_off[i] + (long long)nv0 * 16;
      g.b_last = a.bt_off[i] + ((long long)(a.r_max - 1) * a.d_out + (long long)nv1 * 8) * 2 - 1;
    }
    return g;
  };
  // rank, scale and slice pages of a slot on target i, read from the tables
  auto slot_info = [&](int slot, int i) {
    const PoolView &p = a.pool;
    const SliceGeo g = slice_geo(i);
    return make_int4(p.rank[(long long)slot * p.n_targets + a.tgt[i]], slice_page(p, slot, g.a_first, g.a_last),
                     slice_page(p, slot, g.b_first, g.b_last), a.scales ? __float_as_int(a.scales[slot]) : 0);
  };

  // ---- the item list, and this cluster's work units resolved once: unit k
  // of the cluster (global unit cid + k * ncl = item * n_tgt + target) gets
  // its slot, rows, rank, scale and the physical pages of this CTA's slices,
  // gathered by thread k.  Grouped here from the index vector (for a single
  // target all of it was gathered while grouping), or read from the plan:
  // its header and thread k's item record are read together (the items array
  // has room for items_cap entries), then rank, scale and pages.
  const bool fused = a.ids != nullptr;
  const int NT = a.n_tgt;
  const int32_t *perm = a.perm;
  int n_items;
  int any_bad = 1;  // (plan path: the plan kernel reported empty slots itself)
  int4 rec = make_int4(0, 0, 0, 0), res = make_int4(-1, -1, 0, 0);
  {
    const int u = cid + tid * ncl, item = u / NT, ti = u - item * NT;
    if (fused) {
      n_items = fused_plan(a, S, tid, slice_geo(0), &any_bad);
      perm = S.f_perm;
      if (item < n_items) {
        rec = unpack_item(S.f_items[item]);
        int4 sl;
        if (NT == 1) {
          sl = S.f_slot[rec.y];
        } else {
          sl = slot_info(rec.x, ti);
        }
        rec.w = sl.x;
        res = make_int4(sl.y, sl.z, sl.w, ti);
      }
    } else {
      int4 d = make_int4(0, 0, 0, 0);
      if (item < a.items_cap) d = a.items[item];
      n_items = a.hdr[a.items_hdr];
      if (item < n_items) {
        const int4 sl = slot_info(d.x, ti);
        rec = make_int4(d.x, d.y, d.z, sl.x);
        res = make_int4(sl.y, sl.z, sl.w, ti);
      }
    }
  }
  __syncthreads();  // (the grouping's arrays are read before they are reused)
  S.it_rec[tid] = rec;
  S.it_res[tid] = res;
  __syncthreads();
  const int nk = (MODE == kExpandOnly) ? 0 : (per_i + TV - 1) / TV;
  const int nn = (MODE == kShrinkOnly) ? 0 : (per_o + TV - 1) / TV;
  const int tpi = nk + nn;
  const int n_units = n_items * NT;
  const int my_items = cid < n_units ? (n_units - cid + ncl - 1) / ncl : 0;  // this cluster's units
  const int total = my_items * tpi;
  const int wlen_a = (kv1 - kv0) * 16, wlen_b = (nv1 - nv0) * 16;

  // ---- resolve an item from its gathered record (items beyond the first
  // kDecodeThreads of a cluster, only possible on the plan path, read theirs
  // now); lane L keeps the addresses of rows L / L + 32 of this CTA's weight
  // slices and of activation row L.
  IssueState is;
  is.li = 0;
  is.tt = 0;
  auto resolve = [&](int li) {
    int4 d, sinfo;
    int ti;
    if (li < kDecodeThreads) {
      d = S.it_rec[li];
      const int4 rs = S.it_res[li];
      sinfo = make_int4(d.w, rs.x, rs.y, rs.z);
      ti = rs.w;
    } else {
      const int u = cid + li * ncl, item = u / NT;
      ti = u - item * NT;
      d = fused ? unpack_item(S.f_items[item]) : a.items[item];
      sinfo = slot_info(d.x, ti);
    }
    is.a_off = a.a_off[ti];
    is.bt_off = a.bt_off[ti];
    is.slot = d.x;
    is.m = d.z;
    const float scale = __int_as_float(sinfo.w);
    const int my_row = lane < is.m ? perm[d.y + lane] : 0;
    const uint8_t *wa[2] = {nullptr, nullptr}, *wb[2] = {nullptr, nullptr};
    bool sa = false, sb = false;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = lane + 32 * h;
      if (j < a.r_max) {
        long long room;
        if (MODE != kExpandOnly && wlen_a > 0) {
          const long long off = is.a_off + ((long long)j * a.d_in + (long long)kv0 * 8) * 2;
          if (sinfo.y >= 0) {
            wa[h] = a.pool.base + (long long)sinfo.y * a.pool.page_bytes +
                    (a.pool.log2_page < 0 ? off : off & (a.pool.page_bytes - 1));
          } else {
            wa[h] = pool_addr(a.pool, is.slot, off, &room);
            sa |= (j < sinfo.x) && (wa[h] == nullptr || room < wlen_a);
          }
        }
        if (MODE != kShrinkOnly && wlen_b > 0) {
          const long long off = is.bt_off + ((long long)j * a.d_out + (long long)nv0 * 8) * 2;
          if (sinfo.z >= 0) {
            wb[h] = a.pool.base + (long long)sinfo.z * a.pool.page_bytes +
                    (a.pool.log2_page < 0 ? off : off & (a.pool.page_bytes - 1));
          } else {
            wb[h] = pool_addr(a.pool, is.slot, off, &room);
            sb |= (j < sinfo.x) && (wb[h] == nullptr || room < wlen_b);
          }
        }
      }
    }
    is.r = sinfo.x;
    is.split_a = __any_sync(0xffffffffu, sa);
    is.split_b = __any_sync(0xffffffffu, sb);
    if (!any_bad && lane == 0 && warp == 0 && crank == 0 && is.r == 0 && !a.pool.loaded[is.slot])
      set_status(a.status, LORA_ERR_NOT_LOADED);  // (in-kernel grouping keeps rows of empty slots)
    is.wa0 = (unsigned long long)wa[0];
    is.wa1 = (unsigned long long)wa[1];
    is.wb0 = (unsigned long long)wb[0];
    is.wb1 = (unsigned long long)wb[1];
    is.xrow = a.x ? (unsigned long long)(a.x + (long long)(my_row / a.x_div) * a.ldx + (long long)kv0 * 8) : 0ull;
    is.yrow = a.y ? (unsigned long long)(a.y + (long long)my_row * a.ldy + a.y_col[ti] + (long long)nv0 * 8) : 0ull;
    ItemInfo &I = my_info[li % kItemSlots];
    if (lane < is.m) I.rows[lane] = my_row;
    if (lane == 0) {
      I.m = is.m;
      I.r = is.r;
      I.scale = scale;
      I.ycol = (int)a.y_col[ti];
    }
    __syncwarp();
  };

  // ---- copy this warp's share of the next tile into `stage`: tile row q
  // (weight rows first, then activation rows) belongs to warp q % 8, and lane
  // q / 8 of that warp moves it with one bulk copy (more only where the row
  // crosses a page).  The warp first announces its rows' bytes on the stage's
  // barrier, then the copies count them down as they land.
  auto issue_next = [&](int stage) {
    if (is.tt == 0) resolve(is.li);
    const bool shrink = is.tt < nk;
    const int t_idx = shrink ? is.tt : is.tt - nk;
    const int v_lo = (shrink ? kv0 : nv0) + t_idx * TV;
    const int wv = max(0, min(v_lo + TV, shrink ? kv1 : nv1) - v_lo);
    const int rows = (wv > 0 && is.r > 0 && is.m > 0) ? is.r + is.m : 0;
    uint8_t *buf = S.ring + stage * a.stage_bytes;
    const unsigned long long w0 = shrink ? is.wa0 : is.wb0, w1 = shrink ? is.wa1 : is.wb1;
    const bool split = shrink ? is.split_a : is.split_b;
    const unsigned long long act = shrink ? is.xrow : is.yrow;
    const int q = warp + kConsumerWarps * lane;  // this lane's row of the tile
    const int my_rows = rows > warp ? (rows - warp + kConsumerWarps - 1) / kConsumerWarps : 0;
    const uint32_t bytes = (uint32_t)wv * 16u;
    // row start addresses (lane-held by the resolve step) for this lane's row
    const unsigned long long wsrc_lo = __shfl_sync(0xffffffffu, w0, q & 31);
    const unsigned long long wsrc_hi = __shfl_sync(0xffffffffu, w1, q & 31);
    const unsigned long long asrc = __shfl_sync(0xffffffffu, act, (q - is.r) & 31);
    if (lane == 0) mbar_arrive_expect_tx(&S.full[stage], (uint32_t)my_rows * bytes);
    __syncwarp();
    if (lane < my_rows) {
      if (q < is.r) {
        const long long off = (long long)t_idx * TV * 16;
        if (split) {  // the slice crosses a page: copy it piece by piece
          const long long loff = (shrink ? is.a_off + (long long)q * a.d_in * 2 : is.bt_off + (long long)q * a.d_out * 2) +
                                 (long long)v_lo * 16;
          copy_pool_row(a.pool, is.slot, loff, bytes, buf + q * pitch, &S.full[stage], a.status);
        } else {
          bulk_g2s(buf + q * pitch, reinterpret_cast<const uint8_t *>(q < 32 ? wsrc_lo : wsrc_hi) + off, bytes,
                   &S.full[stage]);
        }
      } else {
        const int i = q - is.r;
        bulk_g2s(buf + act_base + i * pitch, reinterpret_cast<const uint8_t *>(asrc) + (long long)t_idx * TV * 16,
                 bytes, &S.full[stage]);
      }
    }
    if (++is.tt == tpi) {
      is.tt = 0;
      ++is.li;
    }
  };

  // prologue: fill the ring
  for (int k = 0; k < total && k < NS; ++k) issue_next(k);

  bool joined = false;  // start barrier completed (needed before the first push)
  int xi = 0;           // exchange counter
  int c_stage = 0;
  uint32_t c_phase = 0;
  int li = 0, tt = 0, m = 0, r = 0;
  float scale = 0.f;
  float sacc[JB < 2 ? 2 : JB][4];  // this warp's MMA fragment of the item's V so far
  ExpandA<JB> va;                  // the item's V as MMA operand fragments (hi + lo)
  for (int g = 0; g < total; ++g) {
    const int stage = c_stage;
    const uint32_t phase = c_phase;
    if (++c_stage == NS) {
      c_stage = 0;
      c_phase ^= 1u;
    }
    const ItemInfo &I = my_info[li % kItemSlots];
    if (tt == 0) {
      m = I.m;
      r = I.r;
      scale = I.scale;
#pragma unroll
      for (int nt = 0; nt < (JB < 2 ? 2 : JB); ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
    }
    const bool live = r > 0 && m > 0;
    if (MODE == kFused && tt == nk && live) {
      // this CTA's split-K share of v is complete: push it to every CTA of
      // the cluster (itself included), then sum what arrived, in fixed CTA
      // order
      shrink_spill<JB>(sacc, r, m, S.red + warp * recv_slice, lane);
      __syncthreads();
      if (!joined) {
        cluster_wait();
        joined = true;
      }
      const int buf = xi & 1, n = m * r;
      float *recv = S.recv + buf * C * recv_slice;
      if (tid == 0) mbar_arrive_expect_tx(&S.recv_full[buf], (uint32_t)(C * n * 4));
      const uint32_t recv_u = smem_u32(recv + crank * n), bar_u = smem_u32(&S.recv_full[buf]);
      for (int e = tid; e < n; e += kConsumerThreads) {
        float part = 0.f;  // this CTA's share of v[e], summed over the warps in fixed order
        for (int w = 0; w < kConsumerWarps; ++w) part += S.red[w * recv_slice + e];
        for (int c = 0; c < C; ++c) st_async_f32(mapa_u32(recv_u + 4u * e, c), part, mapa_u32(bar_u, c));
      }
      mbar_wait_cluster_bounded(&S.recv_full[buf], (xi >> 1) & 1, a.status);
      for (int e = tid; e < n; e += kConsumerThreads) {
        float sum = 0.f;
        for (int c = 0; c < C; ++c) sum += recv[c * n + e];
        const int i = e / r, j = e - i * r;
        S.v[i * kRMax + j] = sum;
      }
      __syncthreads();
      ++xi;
    }
    const bool ok = mbar_wait_bounded(&S.full[stage], phase, a.status);
    if (MODE == kExpandOnly && tt == 0 && live) {
      for (int idx = tid; idx < m * r; idx += kConsumerThreads) {
        const int i = idx / r, j = idx - i * r;
        S.v[i * kRMax + j] = a.v[(long long)I.rows[i] * a.ldv + j];
      }
      __syncthreads();
    }
    if (ok && live) {
      const uint8_t *buf = S.ring + stage * a.stage_bytes;
      const bool shrink = tt < nk;
      const int t_idx = shrink ? tt : tt - nk;
      const int v_lo = (shrink ? kv0 : nv0) + t_idx * TV;
      const int wv = max(0, min(v_lo + TV, shrink ? kv1 : nv1) - v_lo);
      const uint32_t buf_u = smem_u32(buf);
      if (shrink) {
        shrink_mma<JB>(buf_u, buf_u + act_base, pitch, wv, r, m, sacc, lane, warp);
      } else {
        if (t_idx == 0) expand_prepare<JB>(S.v, r, m, va, lane);
        if (wv > 0)
          expand_mma<JB>(buf_u, buf + act_base, smem_u32(S.zero), pitch, wv, v_lo, r, m, va, scale, I.rows, I.ycol, a,
                         lane, warp);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[stage]);  // this warp is done with the stage
    if (g + NS < total) {                          // refill it once every warp is
      mbar_wait_bounded(&S.empty[stage], phase, a.status);
      issue_next(stage);
    }
    if (MODE == kShrinkOnly && tt == tpi - 1 && live) {
      shrink_spill<JB>(sacc, r, m, S.red + warp * recv_slice, lane);
      __syncthreads();
      if (!joined) {
        cluster_wait();
        joined = true;
      }
      const int buf = xi & 1, n = m * r;
      float *recv = S.recv + buf * C * recv_slice;
      if (tid == 0) mbar_arrive_expect_tx(&S.recv_full[buf], (uint32_t)(C * n * 4));
      const uint32_t recv_u = smem_u32(recv + crank * n), bar_u = smem_u32(&S.recv_full[buf]);
      for (int e = tid; e < n; e += kConsumerThreads) {
        float part = 0.f;
        for (int w = 0; w < kConsumerWarps; ++w) part += S.red[w * recv_slice + e];
        for (int c = 0; c < C; ++c) st_async_f32(mapa_u32(recv_u + 4u * e, c), part, mapa_u32(bar_u, c));
      }
      mbar_wait_cluster_bounded(&S.recv_full[buf], (xi >> 1) & 1, a.status);
      if (crank == 0) {
        for (int idx = tid; idx < m * a.r_max; idx += kConsumerThreads) {
          const int i = idx / a.r_max, j = idx - i * a.r_max;
          float sum = 0.f;
          if (j < r)
            for (int c = 0; c < C; ++c) sum += recv[c * n + i * r + j];
          a.v[(long long)I.rows[i] * a.ldv + j] = sum;
        }
      }
      __syncthreads();
      ++xi;
    }
    if (++tt == tpi) {
      tt = 0;
      ++li;
    }
  }
  if (!joined) cluster_wait();
  // No CTA leaves while a peer may still write into its shared memory.
  cluster_arrive();
  cluster_wait();
}

// Ring geometry for a slot rank: 1 KiB rows and two stages (one shrink and one
// expand tile of a d=4096 item in flight) up to rank 32; 512-byte rows beyond.
static void decode_geometry(int r_max, int *tile_vecs, int *row_pitch, int *n_stages) {
  *tile_vecs = r_max <= 32 ? 64 : 32;
  *row_pitch = *tile_vecs * 16 + 16;
  *n_stages = 2;
}

static int decode_smem_bytes(int r_max, int *stage_bytes, int *n_stages) {
  int tv, pitch;
  decode_geometry(r_max, &tv, &pitch, n_stages);
  *stage_bytes = (r_max + kItemRows) * pitch;
  return *n_stages * *stage_bytes + (2 * kMaxStages + 2) * 8 + 32 + kConsumerWarps * kItemSlots * (int)sizeof(ItemInfo) +
         kConsumerWarps * kItemRows * r_max * 4 + kItemRows * kRMax * 4 + 2 * kClusterCtas * kItemRows * r_max * 4 +
         kFusedBytes;
}

// Rank rows per warp of the shrink: the smallest power of two with
// 8 * JB >= r_max (ranks below r_max use the same kernel).
static int jb_for(int r_max) { return r_max <= 8 ? 1 : r_max <= 16 ? 2 : r_max <= 32 ? 4 : 8; }

template <int MODE, int JB>
static cudaError_t launch_one(const DecodeArgs &a, int csize, int n_clusters, int smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_clusters * csize);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_kernel<MODE, JB>, a);
}

template <int MODE>
static cudaError_t launch_mode(const DecodeArgs &a, int jb, int csize, int n_clusters, int smem, cudaStream_t st) {
  switch (jb) {
    case 1: return launch_one<MODE, 1>(a, csize, n_clusters, smem, st);
    case 2: return launch_one<MODE, 2>(a, csize, n_clusters, smem, st);
    case 4: return launch_one<MODE, 4>(a, csize, n_clusters, smem, st);
    default: return launch_one<MODE, 8>(a, csize, n_clusters, smem, st);
  }
}

template <int MODE, int JB>
static cudaError_t set_smem(int bytes) {
  return cudaFuncSetAttribute(decode_kernel<MODE, JB>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int MODE>
static cudaError_t set_smem_all(int bytes) {
  cudaError_t e = set_smem<MODE, 1>(bytes);
  if (e == cudaSuccess) e = set_smem<MODE, 2>(bytes);
  if (e == cudaSuccess) e = set_smem<MODE, 4>(bytes);
  if (e == cudaSuccess) e = set_smem<MODE, 8>(bytes);
  return e;
}

template <int JB>
static cudaError_t max_clusters(int *n, const cudaLaunchConfig_t *cfg) {
  return cudaOccupancyMaxActiveClusters(n, decode_kernel<kFused, JB>, cfg);
}

int decode_setup(lora_pool *pool) {
  int stage, ns;
  const int smem = decode_smem_bytes(pool->r_max, &stage, &ns);
  pool->decode_smem = smem;
  // The attribute is per function: set it to what the largest rank needs, so
  // that pools of different r_max can coexist.
  const int smem_cap = decode_smem_bytes(kRMax, &stage, &ns);
  if (set_smem_all<kFused>(smem_cap) != cudaSuccess || set_smem_all<kShrinkOnly>(smem_cap) != cudaSuccess ||
      set_smem_all<kExpandOnly>(smem_cap) != cudaSuccess)
    return LORA_ERR_CUDA;
  // co-resident clusters of 8 and of 4 CTAs at this pool's shared memory
  for (int csize : {kClusterCtas, kClusterCtas / 2}) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    cudaError_t e;
    switch (jb_for(pool->r_max)) {
      case 1: e = max_clusters<1>(&n, &cfg); break;
      case 2: e = max_clusters<2>(&n, &cfg); break;
      case 4: e = max_clusters<4>(&n, &cfg); break;
      default: e = max_clusters<8>(&n, &cfg); break;
    }
    if (e != cudaSuccess || n < 1) return LORA_ERR_CUDA;
    if (csize == kClusterCtas) pool->decode_max_clusters = n;
    else pool->decode_max_clusters4 = n;
  }
  return LORA_OK;
}

int launch_decode(lora_pool *pool, int mode, int target, const void *x, int ldx, void *y, int ldy,
                  const float *scales, float *v, int ldv, int T, const void *ws, cudaStream_t st) {
  return launch_decode_items(pool, mode, target, x, ldx, y, ldy, scales, v, ldv, T, ws, st, kHdrItems);
}

static int launch_decode_args(lora_pool *pool, int mode, int n_tgt, const int *targets, const int *y_cols,
                              const void *x, int ldx, void *y, int ldy, const float *scales, float *v, int ldv,
                              int T, const void *ws, const int32_t *ids, cudaStream_t st, int items_hdr,
                              int x_div = 1, const int32_t *moe_topk = nullptr, int moe_k = 0, int moe_e = 0) {
  DecodeArgs a;
  a.pool = pool->view();
  a.d_in = pool->targets[targets[0]].d_in;
  a.d_out = pool->targets[targets[0]].d_out;
  a.r_max = pool->r_max;
  a.n_tgt = n_tgt;
  for (int i = 0; i < kMaxMulti; ++i) {
    const int t = targets[i < n_tgt ? i : 0];
    a.tgt[i] = t;
    a.a_off[i] = pool->a_off[t];
    a.bt_off[i] = pool->bt_off[t];
    a.y_col[i] = (y_cols && i < n_tgt) ? y_cols[i] : 0;
  }
  a.x = static_cast<const uint16_t *>(x);
  a.ldx = ldx;
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.scales = scales;
  if (ids) {
    a.hdr = nullptr;
    a.perm = nullptr;
    a.items = nullptr;
  } else {
    PlanLayout L = plan_layout(T);
    PlanView pv = plan_view(const_cast<void *>(ws), L);
    a.hdr = pv.hdr;
    a.perm = pv.perm;
    a.items = pv.items;
  }
  a.items_cap = ids ? 0 : plan_layout(T).i_max;
  a.ids = ids;
  a.T = T;
  a.x_div = x_div;
  a.moe_topk = moe_topk;
  a.moe_k = moe_k;
  a.moe_e = moe_e;
  a.v = v;
  a.ldv = ldv;
  a.status = pool->d_status;
  a.items_hdr = items_hdr;
  int stage, ns;
  const int smem = decode_smem_bytes(pool->r_max, &stage, &ns);
  a.stage_bytes = stage;
  a.n_stages = ns;
  decode_geometry(pool->r_max, &a.tile_vecs, &a.row_pitch, &ns);
  // Items are bounded by min(T, n_slots) segments plus T / kItemRows chunk
  // splits (times the targets: one work unit per item and target); clusters
  // loop over units, so the grid never exceeds what fits.
  // A batch that may hold more than twice as many items as there are 8-CTA
  // clusters takes 4-CTA clusters: twice the items in flight, each split
  // four ways instead of eight.  (Up to rank 32 only: with rank 64 the
  // 512-byte rows double the tiles of each item and it measured slower.)
  // (The cluster size follows the items of one target, so that a launch over
  // several targets splits each item exactly as a launch per target would:
  // measured, the finer split gave a launch over q, k and v no gain.)
  const long long items1 = (long long)std::min(T, pool->n_slots) + (T + kItemRows - 1) / kItemRows;
  const long long bound = items1 * (long long)n_tgt;
  const bool small_clusters =
      pool->r_max <= 32 && items1 > 2LL * pool->decode_max_clusters && pool->decode_max_clusters4 > 0;
  const int csize = small_clusters ? kClusterCtas / 2 : kClusterCtas;
  int n_clusters = (int)std::min<long long>(
      bound, (long long)(small_clusters ? pool->decode_max_clusters4 : pool->decode_max_clusters));
  if (n_clusters < 1) n_clusters = 1;
  cudaError_t e;
  g_launches.fetch_add(1);
  const int jb = jb_for(pool->r_max);
  if (mode == kFused) e = launch_mode<kFused>(a, jb, csize, n_clusters, smem, st);
  else if (mode == kShrinkOnly) e = launch_mode<kShrinkOnly>(a, jb, csize, n_clusters, smem, st);
  else e = launch_mode<kExpandOnly>(a, jb, csize, n_clusters, smem, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

int launch_decode_items(lora_pool *pool, int mode, int target, const void *x, int ldx, void *y, int ldy,
                        const float *scales, float *v, int ldv, int T, const void *ws, cudaStream_t st,
                        int items_hdr) {
  return launch_decode_args(pool, mode, 1, &target, nullptr, x, ldx, y, ldy, scales, v, ldv, T, ws, nullptr, st,
                            items_hdr);
}

int launch_decode_ids(lora_pool *pool, int mode, int target, const void *x, int ldx, void *y, int ldy,
                      const float *scales, float *v, int ldv, const int32_t *ids, int T, cudaStream_t st) {
  if (T < 1 || T > kFusedMaxT) return LORA_ERR_INVALID_ARG;
  return launch_decode_args(pool, mode, 1, &target, nullptr, x, ldx, y, ldy, scales, v, ldv, T, nullptr, ids, st,
                            kHdrItems);
}

int launch_decode_moe(lora_pool *pool, int target, const void *x, int ldx, void *y, int ldy, const float *scales,
                      const int32_t *lora_ids, const int32_t *topk, int n_pairs, int top_k, int n_experts,
                      const void *ws, cudaStream_t st) {
  if (!ws) {  // pairs grouped inside the kernel from the routing itself
    if (n_pairs < 1 || n_pairs > kFusedMaxT) return LORA_ERR_INVALID_ARG;
    return launch_decode_args(pool, kFused, 1, &target, nullptr, x, ldx, y, ldy, scales, nullptr, 0, n_pairs,
                              nullptr, lora_ids, st, kHdrItems, top_k, topk, top_k, n_experts);
  }
  // the pairs' slots were planned into ws (lora_plan_ids over them)
  return launch_decode_args(pool, kFused, 1, &target, nullptr, x, ldx, y, ldy, scales, nullptr, 0, n_pairs, ws,
                            nullptr, st, kHdrItems, top_k);
}

int launch_decode_multi(lora_pool *pool, int n_tgt, const int *targets, const int *y_cols, const void *x, int ldx,
                        void *y, int ldy, const float *scales, const int32_t *ids, int T, const void *ws,
                        cudaStream_t st) {
  if (n_tgt < 1 || n_tgt > kMaxMulti || (ids && (T < 1 || T > kFusedMaxT))) return LORA_ERR_INVALID_ARG;
  return launch_decode_args(pool, kFused, n_tgt, targets, y_cols, x, ldx, y, ldy, scales, nullptr, 0, T, ws, ids,
                            st, kHdrItems);
}

}  // namespace lora
