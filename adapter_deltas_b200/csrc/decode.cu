// decode.cu -- decode path of the multi-LoRA delta: one launch for every
// adapter of a batch.
//
// For the rows t of adapter a the kernel computes
//     v = A_a x[t]                 (shrink: r_a dot products of length d_in)
//     y[t] += (alpha_a / r_a) B_a v (expand, fused with the scale and the
//                                   in-place accumulate)
// which is the per-request term of y = xW + (x A_i) B_i (alpha / r) on
// "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU" (section "Why can't you
// just merge LoRA weights into the base model?").  The cost the same page
// gives for a mixed batch is the adapters' weight bytes (section "How does one
// batch run 30 different adapters at once?"), so the kernel is built to keep
// HBM busy with as few dependent steps as possible.
//
// Work.  Rows are grouped by adapter into items of up to kItemRows rows (in
// the kernel itself for batches up to kFusedMaxT rows, else by the plan
// kernel).  A work unit is one item on one target and one range of d_out
// columns: it streams the item's whole A slice with its rows of x (the
// shrink, v in registers), then the B^T columns and y rows of its range (the
// expand).  The shrink / expand split of "Multi-LoRA Serving: Sharing One GPU
// Across Adapters" (section "MoE Models Raise the Bar") is kept inside the
// unit: when an item is cut into several column ranges, each of its units
// computes v itself (the A slice is then read from HBM once and from L2 by
// the others), so units never wait on one another -- no grid-wide
// synchronisation, no scratch memory, and every row's v is summed in the same
// fixed order whatever the batch, the path or the launch.
//
// Column ranges per item: enough for about one unit per CTA, uniform over the
// items; when that still leaves SMs idle, items of many rows (whose expand
// tiles carry many y rows) get twice as many (uneven_ranges).
//
// B200 mapping.  Per CTA one producer warp walks the CTA's units and streams
// their tiles into a shared-memory ring with 1-D bulk async copies
// (cp.async.bulk, no multicast): the first r rows of an adapter tile are one
// contiguous range of the pool's tiled block (one copy), activation rows one
// copy each; the copies complete on mbarriers.  Eight consumer warps run the
// contractions on warp-level bf16 MMA (a full tile on a compile-time
// schedule), update the staged y rows in place with ldmatrix / stmatrix and
// send them out -- coalesced stores for small items, one bulk copy per row
// for larger ones.  The producer runs up to the ring depth ahead of them.
#include <algorithm>
#include <climits>

#include "internal.cuh"

namespace lora {

constexpr int kProdWarp = kConsumerWarps;  // copies the units' tiles into the ring
constexpr int kDecWarps = kConsumerWarps + 1;
constexpr int kDecThreads = kDecWarps * 32;
// CTAs per SM the kernel is compiled for: ranks 9..16 take 1024-column tiles
// whose ring fills one SM's shared memory (one CTA, registers to spare); the
// other ranks' rings fit twice.
constexpr int dec_min_blocks(int jb) { return jb == 2 ? 1 : 2; }
// 16-byte chunks per row of a full pool tile for the kernel's rank class
// (the tile width of the largest rank the class serves).
__host__ __device__ constexpr int full_tile_chunks(int jb) { return pool_tile_cols(8 * jb) / 8; }
// Items of up to this many rows write their y rows back with plain stores;
// larger ones with bulk copies.
constexpr int kStoreRowsMax = 4;
constexpr int kCacheItems = 256;  // items whose records a CTA keeps in shared memory
constexpr int kCachePerm = 512;   // grouped row positions a CTA keeps in shared memory

enum UnitKind : int { kUnitShrink = 0, kUnitExpand = 1, kUnitEnd = 2 };

// What a unit needs in the consumers, written once per unit by the producer
// into a small ring of records (a record is reused only after all the stages
// that name it have been released).
struct UnitRec {
  int m, r, ycol;
  float scale;
  int rows[kItemRows];
};
constexpr int kRecs = kMaxStages + 1;

// What a stage holds: its kind and flags, where its tile starts, its width,
// and the unit record -- one 16-byte word written by the producer before it
// arrives on the stage's full barrier (the consumers read it after their
// wait).  kind | first << 4 | last << 5 | rec << 8.
struct StageHdr {
  int bits, v_lo, wv, pad;
};

struct DecodeArgs {
  PoolView pool;
  int d_in, d_out, r_max;
  // targets of this launch: all share x, d_in and d_out; target i writes its
  // delta into columns y_col[i] .. y_col[i] + d_out - 1 of y
  int n_tgt;
  int tgt[kMaxMulti];
  long long a_off[kMaxMulti], bt_off[kMaxMulti], y_col[kMaxMulti];
  const uint16_t *x;
  long long ldx;
  uint16_t *y;
  long long ldy;
  const float *scales;
  // plan path
  const int32_t *hdr;
  int early;  // plan path (not expand-only, T <= kCachePerm): see early_prefetch
  const int32_t *perm;
  const int4 *items;
  int items_hdr;  // header word holding the item count to process
  int items_cap;  // entries the plan's items array has room for
  // in-kernel grouping (ids non-null, T <= kFusedMaxT)
  const int32_t *ids;
  int T;
  int x_div;  // row t reads x row t / x_div (1; top_k for routed expert pairs)
  // routed expert pairs (moe_topk non-null): row p is the pair (token p /
  // moe_k, its (p % moe_k)-th expert), ids[] holds each token's adapter, and
  // the pair's slot is adapter * moe_e + expert
  const int32_t *moe_topk;
  int moe_k, moe_e;
  float *v;  // shrink-only: output [T, ldv]; expand-only: input
  long long ldv;
  int n_sms;  // SMs of the device
  int stall;  // test only: the producer fills no stage
  int *status;
  unsigned long long wait_ns;
  int kcv;        // 16-byte chunks per full tile row (the pool's tile width)
  int pitch;      // bytes between staged activation rows (kcv * 16 + 16)
  int stage_bytes;
  int n_stages;
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
__device__ __forceinline__ void stsm_x4(uint32_t addr, const uint32_t (&r)[4]) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Staged weight tile: row j of a tile with `wv` chunks per row starts at
// j * wv * 16, and its chunk c sits at swz_chunk(c, j, wv) (the pool's own
// arrangement, copied as it is).
__device__ __forceinline__ uint32_t wt_addr(uint32_t buf_u, int j, int c, int wv) {
  return buf_u + (uint32_t)(j * wv + swz_chunk(c, j, wv)) * 16u;
}

// Shrink: this warp's share of V[i][j] = sum_k x[i][k] A[j][k] over the
// tile's columns, accumulated in acc[n-tile][4] (rows g, g + 8 and columns
// 2t, 2t + 1 of each 8-rank n-tile; g = lane / 4, t = lane % 4).  The warps
// split the tile's 16-column k-steps (warp w: k-steps w, w + 8, ...); within a
// tile the warp's k-steps go two at a time into two accumulator sets, added
// at the end of the tile in fixed order, so that the MMA latency chains
// overlap.  Rows i >= m and ranks j >= r read row 0 of their operand instead:
// an output element depends only on its own row of each operand, so those
// lanes' results are simply never spilled.  An odd last chunk (8 columns)
// zeroes both operands' upper k half.
template <int JB>
__device__ __forceinline__ void shrink_mma(uint32_t buf_u, uint32_t act_u, int pitch, int wv, int r, int m,
                                           float (&acc)[JB < 2 ? 2 : JB][4], int lane, int warp) {
  constexpr int NT = JB < 2 ? 2 : JB;  // 8-rank n-tiles (loaded two at a time)
  constexpr int NP = NT / 2;
  const int ksteps = (wv + 1) / 2;     // 16 columns = two 16-byte chunks
  const int xr = (lane & 7) + ((lane >> 3) & 1) * 8, xk = (lane >> 4) * 16;
  const uint32_t xrow = act_u + (xr < m ? xr : 0) * pitch + xk;
  int arow[NP], ax[NP];
  uint32_t abase[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int j = (lane & 7) + (lane >> 4) * 8 + 16 * p;
    arow[p] = j < r ? j : 0;
    abase[p] = buf_u + (uint32_t)(arow[p] * wv) * 16u;
    ax[p] = arow[p] & 7;
  }
  const int ahalf = (lane >> 3) & 1;
  const int np = min(NP, (r + 15) >> 4);  // 16-rank blocks within the adapter's rank
  int ks = warp;
  if (NP <= 2) {
    // k-steps whose two chunks lie in a complete group of eight (chunk c at
    // c ^ (row % 8)), two per pass
    const int nk_full = (wv & ~7) >> 1;
    float acc2[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc2[nt][0] = acc2[nt][1] = acc2[nt][2] = acc2[nt][3] = 0.f;
    for (; ks + kConsumerWarps < nk_full; ks += 2 * kConsumerWarps) {
      const int k1 = ks + kConsumerWarps;
      uint32_t a0[4], a1[4], b0[NP][4], b1[NP][4];
      ldsm_x4(xrow + ks * 32, a0);
      ldsm_x4(xrow + k1 * 32, a1);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        if (p < np) {
          ldsm_x4(abase[p] + ((uint32_t)((2 * ks + ahalf) ^ ax[p]) << 4), b0[p]);
          ldsm_x4(abase[p] + ((uint32_t)((2 * k1 + ahalf) ^ ax[p]) << 4), b1[p]);
        }
      }
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        if (p < np) {
          mma_bf16_16816(acc[2 * p], a0, b0[p][0], b0[p][1]);
          mma_bf16_16816(acc[2 * p + 1], a0, b0[p][2], b0[p][3]);
          mma_bf16_16816(acc2[2 * p], a1, b1[p][0], b1[p][1]);
          mma_bf16_16816(acc2[2 * p + 1], a1, b1[p][2], b1[p][3]);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      acc[nt][0] += acc2[nt][0];
      acc[nt][1] += acc2[nt][1];
      acc[nt][2] += acc2[nt][2];
      acc[nt][3] += acc2[nt][3];
    }
  }
  // the rest one k-step at a time (a trailing partial group, an odd last chunk)
  for (; ks < ksteps; ks += kConsumerWarps) {
    const bool half = 2 * ks + 1 >= wv;
    uint32_t a[4];
    ldsm_x4(xrow + ks * 32, a);
    if (half) a[2] = a[3] = 0u;
    // an odd last chunk: the upper-half lanes read chunk 2ks again (zeroed below)
    const int c = half ? 2 * ks : 2 * ks + ahalf;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      if (p >= np) break;
      uint32_t b[4];
      ldsm_x4(wt_addr(buf_u, arow[p], c, wv), b);
      if (half) b[1] = b[3] = 0u;
      mma_bf16_16816(acc[2 * p], a, b[0], b[1]);
      mma_bf16_16816(acc[2 * p + 1], a, b[2], b[3]);
    }
  }
}

// The same over a full tile (wv = the pool's tile width, every chunk in a
// complete group of eight): the warp's KPW k-steps have compile-time
// positions; their operands are loaded in batches of k-steps (four; two
// for ranks past 16, one past 32) ahead of the MMAs, and consecutive k-steps alternate between two
// accumulator sets (added at the end, in fixed order; ranks up to 32 --
// beyond, the warp's two k-steps have eight chains already).
template <int JB, int KPW>
__device__ __forceinline__ void shrink_full(uint32_t buf_u, uint32_t act_u, int pitch, int wv, int r, int m,
                                            float (&acc)[JB < 2 ? 2 : JB][4], int lane, int warp) {
  constexpr int NT = JB < 2 ? 2 : JB;
  constexpr int NP = NT / 2;
  constexpr int BATCH = NP >= 4 ? 1 : NP >= 2 ? 2 : KPW < 4 ? KPW : 4;  // k-steps whose operands load together
  const int xr = (lane & 7) + ((lane >> 3) & 1) * 8, xk = (lane >> 4) * 16;
  const uint32_t xrow = act_u + (xr < m ? xr : 0) * pitch + xk;
  const int ahalf = (lane >> 3) & 1;
  uint32_t abase[NP], ax[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int j = (lane & 7) + (lane >> 4) * 8 + 16 * p;
    const int jr = j < r ? j : 0;
    abase[p] = buf_u + (uint32_t)(jr * wv) * 16u;
    ax[p] = (uint32_t)(jr & 7);
  }
  const int np = min(NP, (r + 15) >> 4);
  float acc2[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc2[nt][0] = acc2[nt][1] = acc2[nt][2] = acc2[nt][3] = 0.f;
#pragma unroll
  for (int b0 = 0; b0 < KPW; b0 += BATCH) {
    uint32_t xa[BATCH][4], wa[BATCH][NP][4];
#pragma unroll
    for (int i = 0; i < BATCH; ++i) ldsm_x4(xrow + (warp + kConsumerWarps * (b0 + i)) * 32, xa[i]);
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      const uint32_t c = (uint32_t)(2 * (warp + kConsumerWarps * (b0 + i)) + ahalf);
#pragma unroll
      for (int p = 0; p < NP; ++p)
        if (p < np) ldsm_x4(abase[p] + ((c ^ ax[p]) << 4), wa[i][p]);
    }
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      float(&dst)[NT][4] = (NT <= 4 && ((b0 + i) & 1)) ? acc2 : acc;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        if (p < np) {
          mma_bf16_16816(dst[2 * p], xa[i], wa[i][p][0], wa[i][p][1]);
          mma_bf16_16816(dst[2 * p + 1], xa[i], wa[i][p][2], wa[i][p][3]);
        }
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    acc[nt][0] += acc2[nt][0];
    acc[nt][1] += acc2[nt][1];
    acc[nt][2] += acc2[nt][2];
    acc[nt][3] += acc2[nt][3];
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
// of each fp32 value), built in registers once per unit; B^T rows are loaded
// transposed by ldmatrix.  Warp w takes the 16-column groups w, w + 8, ...
template <int JB>
struct ExpandA {
  static constexpr int KS = JB < 2 ? 1 : JB / 2;  // 16-rank k-steps
  uint32_t hi[KS][4], lo[KS][4];
};

// s_v: V of the unit's rows, row i at s_v + i * ld.
template <int JB>
__device__ __forceinline__ void expand_prepare(const float *s_v, int ld, int r, int m, ExpandA<JB> &A, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < ExpandA<JB>::KS; ++ks) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // a0: (g, 2t), a1: (g+8, 2t), a2: (g, 2t+8), a3: (g+8, 2t+8)
      const int i = g + (q & 1) * 8, j = 16 * ks + 2 * t + (q >> 1) * 8;
      const float v0 = (i < m && j < r) ? s_v[i * ld + j] : 0.f;
      const float v1 = (i < m && j + 1 < r) ? s_v[i * ld + j + 1] : 0.f;
      const uint32_t h = pack_bf16x2(v0, v1);
      A.hi[ks][q] = h;
      A.lo[ks][q] = pack_bf16x2(v0 - bf16_lo(h), v1 - bf16_hi(h));
    }
  }
}

// Per-lane addressing of one expand tile, set up once per tile.  Lane
// (g = lane / 4, t = lane % 4) owns output rows g and g + 8 and, in every
// 8-column n-tile, columns 2t and 2t + 1; its ldmatrix row is rank
// 16 ks + bj of chunk half bc.
struct ExpandLane {
  uint32_t rb[4];        // per 16-rank block: the lane's B^T row (or 16 zero bytes past the rank)
  uint32_t xm[4], cm[4]; // its swizzle (row % 8) and chunk mask (0 for the zero row)
  uint8_t *ys0, *ys1;    // staged y of rows g, g + 8 at column 2t (updated in place)
  bool ok0, ok1;         // rows g, g + 8 belong to the item
  int bc, nks;
};

template <int JB>
__device__ __forceinline__ ExpandLane expand_lane(uint32_t buf_u, uint8_t *yb, uint32_t zero_u, int pitch, int wv,
                                                  int r, int m, int lane) {
  ExpandLane L;
  const int g = lane >> 2, t = lane & 3;
  const int bj = (lane & 7) + ((lane >> 3) & 1) * 8;
  L.bc = lane >> 4;
#pragma unroll
  for (int ks = 0; ks < ExpandA<JB>::KS; ++ks) {
    // ranks j >= r read 16 zero bytes: their V is zero and stale weights
    // (possibly not finite) must not meet it
    const int j = 16 * ks + bj;
    const bool ok = j < r;
    L.rb[ks] = ok ? buf_u + (uint32_t)(j * wv) * 16u : zero_u;
    L.xm[ks] = ok ? (uint32_t)(j & 7) : 0u;
    L.cm[ks] = ok ? 0xffffffffu : 0u;
  }
  L.nks = (r + 15) >> 4;
  L.ys0 = yb + g * pitch + 4 * t;
  L.ys1 = L.ys0 + 8 * pitch;
  L.ok0 = g < m;
  L.ok1 = g + 8 < m;
  return L;
}

// Staged y[row][col .. col + 1] += scale * (d0, d1) for the lane's two rows
// (the rows go to global memory afterwards, one bulk copy each).
__device__ __forceinline__ void expand_store(const ExpandLane &L, int col, const float (&d)[4], float scale) {
  if (L.ok0) {
    uint32_t *p = reinterpret_cast<uint32_t *>(L.ys0 + col * 2);
    const uint32_t yv = *p;
    *p = pack_bf16x2(fmaf(scale, d[0], bf16_lo(yv)), fmaf(scale, d[1], bf16_hi(yv)));
  }
  if (L.ok1) {
    uint32_t *p = reinterpret_cast<uint32_t *>(L.ys1 + col * 2);
    const uint32_t yv = *p;
    *p = pack_bf16x2(fmaf(scale, d[2], bf16_lo(yv)), fmaf(scale, d[3], bf16_hi(yv)));
  }
}

// G complete 16-column groups cg0, cg0 + 8, ... (their chunks lie in complete
// groups of eight, so chunk c of rank row j sits at c ^ (j % 8)).  Each
// group's accumulator takes, per 16-rank block, the hi term and then the lo
// term; the G chains overlap.
template <int JB, int G>
__device__ __forceinline__ void expand_pass(const ExpandLane &L, const ExpandA<JB> &A, float scale, int cg0) {
  float acc[G][2][4];
#pragma unroll
  for (int q = 0; q < G; ++q)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) acc[q][nt][0] = acc[q][nt][1] = acc[q][nt][2] = acc[q][nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < ExpandA<JB>::KS; ++ks) {
    if (ks < L.nks) {
      uint32_t b[G][4];
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const uint32_t c = (uint32_t)(2 * (cg0 + q * kConsumerWarps) + L.bc);
        ldsm_x4_t(L.rb[ks] + (((c ^ L.xm[ks]) & L.cm[ks]) << 4), b[q]);
      }
#pragma unroll
      for (int q = 0; q < G; ++q) {
        mma_bf16_16816(acc[q][0], A.hi[ks], b[q][0], b[q][1]);
        mma_bf16_16816(acc[q][1], A.hi[ks], b[q][2], b[q][3]);
      }
#pragma unroll
      for (int q = 0; q < G; ++q) {
        mma_bf16_16816(acc[q][0], A.lo[ks], b[q][0], b[q][1]);
        mma_bf16_16816(acc[q][1], A.lo[ks], b[q][2], b[q][3]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < G; ++q) {
    const int col = (cg0 + q * kConsumerWarps) * 16;
    expand_store(L, col, acc[q][0], scale);
    expand_store(L, col + 8, acc[q][1], scale);
  }
}

// One group of a partial chunk group at the tile's end (chunks unswizzled;
// an odd last chunk is half a group: 8 columns).
template <int JB>
__device__ __forceinline__ void expand_tail(const ExpandLane &L, const ExpandA<JB> &A, float scale, uint32_t zero_u,
                                            int wv, int cg) {
  float acc[2][4] = {};
  const bool half = 2 * cg + 1 >= wv;
  const uint32_t c = (uint32_t)((half && L.bc) ? 2 * cg : 2 * cg + L.bc);
#pragma unroll
  for (int ks = 0; ks < ExpandA<JB>::KS; ++ks) {
    if (ks < L.nks) {
      uint32_t b[4];
      ldsm_x4_t(L.cm[ks] ? L.rb[ks] + (c << 4) : zero_u, b);
      mma_bf16_16816(acc[0], A.hi[ks], b[0], b[1]);
      mma_bf16_16816(acc[1], A.hi[ks], b[2], b[3]);
      mma_bf16_16816(acc[0], A.lo[ks], b[0], b[1]);
      mma_bf16_16816(acc[1], A.lo[ks], b[2], b[3]);
    }
  }
  expand_store(L, cg * 16, acc[0], scale);
  if (!half) expand_store(L, cg * 16 + 8, acc[1], scale);
}

// A full tile (wv = the pool's tile width): the warp's GPW column groups
// warp, warp + 8, ... in passes of G, every B^T operand of a pass loaded
// before its MMAs; the staged y of a group (rows 0..15, its 16 columns) is
// read and written back with one ldmatrix / stmatrix each, in the MMA
// fragment layout (rows past the item are staging rows nobody stores).
template <int JB, int GPW, int G>
__device__ __forceinline__ void expand_full(const ExpandLane &L, const ExpandA<JB> &A, float scale, uint32_t yb_u,
                                            int pitch, int lane, int warp) {
  // ldmatrix / stmatrix row of this lane in a group's staged y
  const uint32_t ylane = yb_u + (uint32_t)(((lane & 7) + ((lane >> 3) & 1) * 8) * pitch + (lane >> 4) * 16);
#pragma unroll
  for (int g0 = 0; g0 < GPW; g0 += G) {
    float acc[G][2][4];
#pragma unroll
    for (int q = 0; q < G; ++q)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) acc[q][nt][0] = acc[q][nt][1] = acc[q][nt][2] = acc[q][nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < ExpandA<JB>::KS; ++ks) {
      if (ks < L.nks) {
        uint32_t b[G][4];
#pragma unroll
        for (int q = 0; q < G; ++q) {
          const uint32_t c = (uint32_t)(2 * (warp + kConsumerWarps * (g0 + q)) + L.bc);
          ldsm_x4_t(L.rb[ks] + (((c ^ L.xm[ks]) & L.cm[ks]) << 4), b[q]);
        }
#pragma unroll
        for (int q = 0; q < G; ++q) {
          mma_bf16_16816(acc[q][0], A.hi[ks], b[q][0], b[q][1]);
          mma_bf16_16816(acc[q][1], A.hi[ks], b[q][2], b[q][3]);
        }
#pragma unroll
        for (int q = 0; q < G; ++q) {
          mma_bf16_16816(acc[q][0], A.lo[ks], b[q][0], b[q][1]);
          mma_bf16_16816(acc[q][1], A.lo[ks], b[q][2], b[q][3]);
        }
      }
    }
    uint32_t yv[G][4];
#pragma unroll
    for (int q = 0; q < G; ++q) ldsm_x4(ylane + (uint32_t)(warp + kConsumerWarps * (g0 + q)) * 32u, yv[q]);
#pragma unroll
    for (int q = 0; q < G; ++q) {
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {  // e: (row g | g + 8) x (n-tile 0 | 1) as ldmatrix orders them
        const float *d = &acc[q][e >> 1][(e & 1) * 2];
        o[e] = pack_bf16x2(fmaf(scale, d[0], bf16_lo(yv[q][e])), fmaf(scale, d[1], bf16_hi(yv[q][e])));
      }
      stsm_x4(ylane + (uint32_t)(warp + kConsumerWarps * (g0 + q)) * 32u, o);
    }
  }
}

// The warp takes the 16-column groups warp, warp + 8, ...: several at a time
// while they lie in complete chunk groups (four for ranks up to 16, two up to
// 32, one beyond: the larger ranks give each group more MMAs of its own),
// then the rest one by one.
template <int JB>
__device__ __forceinline__ void expand_mma(uint32_t buf_u, uint8_t *yb, uint32_t zero_u, int pitch, int wv, int r,
                                           int m, const ExpandA<JB> &A, float scale, int lane, int warp) {
  constexpr int G = JB <= 2 ? 4 : JB == 4 ? 2 : 1;
  const ExpandLane L = expand_lane<JB>(buf_u, yb, zero_u, pitch, wv, r, m, lane);
  if (wv == full_tile_chunks(JB)) {
    constexpr int GPW = full_tile_chunks(JB) / 2 / kConsumerWarps;  // column groups per warp
    expand_full<JB, GPW, JB == 2 ? GPW : G>(L, A, scale, smem_u32(yb), pitch, lane, warp);
    return;
  }
  const int groups = (wv + 1) / 2;       // 16-column groups (an odd last chunk is half a group)
  const int full = (wv & ~7) >> 1;       // groups inside complete chunk groups of eight
  int cg = warp;
  for (; cg + (G - 1) * kConsumerWarps < full; cg += G * kConsumerWarps) expand_pass<JB, G>(L, A, scale, cg);
  if (G > 1)
    for (; cg < full; cg += kConsumerWarps) expand_pass<JB, 1>(L, A, scale, cg);
  for (; cg < groups; cg += kConsumerWarps) expand_tail<JB>(L, A, scale, zero_u, wv, cg);
}

// ------------------------------------------------------------ sync helpers
// Named barrier 1 over the eight consumer warps (the producer warp never
// joins it).
__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory"); }
// The same barrier, returning whether `pred` held in every consumer thread.
__device__ __forceinline__ bool cons_sync_and(bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)pred), "n"(kConsumerThreads)
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Generic-proxy writes to shared memory that a later bulk copy will
// overwrite: order them before the async proxy's accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ shared memory
struct DecSmem {
  uint8_t *ring;
  StageHdr *hdr;          // [kMaxStages]
  UnitRec *rec;           // [kRecs]
  uint64_t *full, *empty; // [kMaxStages] each
  uint8_t *zero;          // 32 zero bytes: the expand's operand rows beyond the rank
  float *v;               // [kItemRows][r_max]: V of the current unit
  int *misc;              // [0]: abort flag; [2]: early_prefetch's decision
  int4 *c_item;           // [kCacheItems]: slot, first grouped position, rows
  int4 *c_slot;           // [kCacheItems]: rank, A page, B^T page, scale bits (first target)
  int *c_perm;            // [kCachePerm]: row of each grouped position
  int *c_pref;            // [kCacheItems + 1]: column ranges of the items before each (uneven ranges)
  long long *tg;          // [3][kMaxMulti]: the launch's targets' A offset, B^T offset, first y column
  // in-kernel grouping temporaries, inside the ring (unused until the
  // grouping is done)
  int *g_key;        // [kGroupTable] hash table of the batch's slots (-1: empty)
  int *g_cnt;        // [kGroupTable][kConsumerWarps] rows of each table entry in each row warp
  uint32_t *g_bits;  // [kGroupTable] bitmap of the slots present
  int *g_bpre;       // [kGroupTable] set bits before each bitmap word
  int *g_dtot;       // [kFusedMaxT] rows of the d-th smallest slot present
  int *g_dseg;       // [kFusedMaxT] its first grouped position
  int *g_ditem;      // [kFusedMaxT] its first item
  int *g_hd;         // [kGroupTable] table entry -> d
  int *g_scan;       // [16] block scan scratch
};

constexpr int kGroupTable = 512;     // hash table entries (>= 2 * kFusedMaxT); bitmap words (kMaxSlots / 32)
constexpr int kRingMin = 40 * 1024;  // room for the grouping temporaries

constexpr int dec_extra_bytes(int r_max) {
  return kMaxStages * (int)sizeof(StageHdr) + kRecs * (int)sizeof(UnitRec) + 2 * kMaxStages * 8 + 64 +
         kItemRows * r_max * 4 + 64 + kCacheItems * 32 + kCachePerm * 4 + 3 * kMaxMulti * 8 +
         (kCacheItems + 4) * 4;
}

__device__ __forceinline__ DecSmem dec_carve(uint8_t *smem, const DecodeArgs &a) {
  DecSmem S;
  uint8_t *p = smem;
  S.ring = p; p += max(a.n_stages * a.stage_bytes, kRingMin);
  S.hdr = reinterpret_cast<StageHdr *>(p); p += kMaxStages * sizeof(StageHdr);
  S.rec = reinterpret_cast<UnitRec *>(p); p += kRecs * sizeof(UnitRec);
  S.full = reinterpret_cast<uint64_t *>(p); p += kMaxStages * 8;
  S.empty = reinterpret_cast<uint64_t *>(p); p += kMaxStages * 8;
  S.zero = p; p += 64;
  S.v = reinterpret_cast<float *>(p); p += kItemRows * a.r_max * 4;
  S.misc = reinterpret_cast<int *>(p); p += 64;
  S.c_item = reinterpret_cast<int4 *>(p); p += kCacheItems * 16;
  S.c_slot = reinterpret_cast<int4 *>(p); p += kCacheItems * 16;
  S.c_perm = reinterpret_cast<int *>(p); p += kCachePerm * 4;
  S.tg = reinterpret_cast<long long *>(p); p += 3 * kMaxMulti * 8;
  S.c_pref = reinterpret_cast<int *>(p);
  uint8_t *q = S.ring;
  S.g_key = reinterpret_cast<int *>(q); q += kGroupTable * 4;
  S.g_cnt = reinterpret_cast<int *>(q); q += kGroupTable * kConsumerWarps * 4;
  S.g_bits = reinterpret_cast<uint32_t *>(q); q += kGroupTable * 4;
  S.g_bpre = reinterpret_cast<int *>(q); q += kGroupTable * 4;
  S.g_dtot = reinterpret_cast<int *>(q); q += kFusedMaxT * 4;
  S.g_dseg = reinterpret_cast<int *>(q); q += kFusedMaxT * 4;
  S.g_ditem = reinterpret_cast<int *>(q); q += kFusedMaxT * 4;
  S.g_hd = reinterpret_cast<int *>(q); q += kGroupTable * 4;
  S.g_scan = reinterpret_cast<int *>(q);
  return S;
}

// ------------------------------------------------------------ grouping
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

// Exclusive scan of one int per thread over the whole block; *total gets
// the sum.  Every thread of the block must call it.
__device__ __forceinline__ int block_scan_excl(int v, int *scratch, int *total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kDecWarps; ++w) {
    const int c = scratch[w];
    base += w < warp ? c : 0;
    tot += c;
  }
  __syncthreads();
  *total = tot;
  return base + incl - v;
}

// Grouping of an index vector inside the kernel, for batches of at most
// kFusedMaxT rows (every CTA computes the same result): the rows of each
// loaded slot in ascending row order, slots in ascending order, cut into
// items of at most kItemRows rows -- the plan kernel's items, in the same
// order.  A row's grouped position is the rows of smaller slots (a bitmap of
// the slots present ranks them) plus the rows of its own slot before it: the
// same slot in earlier warps (per-warp counts kept in a small hash table of
// the batch's slots) and in its own warp (match_any).  Each row's thread also
// loads what the first target needs of its slot (rank, the pages of its A and
// B^T blocks, scale) while the ids are still arriving; an item's first row
// stores them.  Rows with a bad id or an empty slot are left out and
// reported, as the plan kernel does.  Fills c_item, c_slot, c_perm; returns
// the item count.
__device__ int fused_group(const DecodeArgs &a, const DecSmem &S, int tid) {
  const int T = a.T, lane = tid & 31, warp = tid >> 5;
  const int n_words = (a.pool.n_slots + 31) >> 5;
  for (int i = tid; i < kGroupTable; i += kDecThreads) S.g_key[i] = -1;
  for (int i = tid; i < kGroupTable * kConsumerWarps; i += kDecThreads) S.g_cnt[i] = 0;
  for (int i = tid; i < n_words; i += kDecThreads) S.g_bits[i] = 0u;
  // The slot's record loads stay in flight through the grouping: only the
  // thread that records an item uses them.  A slot that is not loaded still
  // forms its items; they get rank 0 and are skipped (rows untouched).
  int key = -1, bad = 0;
  int ld = 1, rk = 0, pa = -1, pb = -1, sc = 0;
  if (tid < T) {
    const int id = a.moe_topk ? moe_pair_slot(a, tid) : a.ids[tid];
    if (id != -1) {
      if (id < -1 || id >= a.pool.n_slots) {
        bad = 1;
      } else {
        const PoolView &p = a.pool;
        key = id;
        ld = p.loaded[id];
        rk = p.rank[(long long)id * p.n_targets + a.tgt[0]];
        pa = block_page(p, id, a.a_off[0], (long long)a.r_max * a.d_in * 2);
        pb = block_page(p, id, a.bt_off[0], (long long)a.r_max * a.d_out * 2);
        sc = a.scales ? __float_as_int(a.scales[id]) : 0;
      }
    }
  }
  const int any_bad = __syncthreads_or(bad);  // (also orders the clearing above before the inserts)
  if (blockIdx.x == 0 && tid == 0) {
    if (any_bad) set_status(a.status, LORA_ERR_BAD_ID);
  }
  // (1) the slot into the hash table (at most kFusedMaxT keys in twice as
  // many entries) and the bitmap
  int h = -1;
  if (key >= 0) {
    h = (int)(((unsigned)key * 2654435761u) >> 23) & (kGroupTable - 1);
    while (true) {
      const int prev = atomicCAS(&S.g_key[h], -1, key);
      if (prev == -1 || prev == key) break;
      h = (h + 1) & (kGroupTable - 1);
    }
    atomicOr(&S.g_bits[key >> 5], 1u << (key & 31));
  }
  // (2) rows of the same slot in this warp, and those before this row
  int wrank = 0;
  if (warp < kConsumerWarps) {
    const unsigned peers = __match_any_sync(0xffffffffu, key >= 0 ? key : -2 - lane);
    wrank = __popc(peers & ((1u << lane) - 1u));
    if (key >= 0 && wrank == 0) S.g_cnt[h * kConsumerWarps + warp] = __popc(peers);
  }
  __syncthreads();
  // (3) set bits before each bitmap word (thread t: words 2t, 2t + 1)
  {
    const int w0 = 2 * tid;
    const int c0 = w0 < n_words ? __popc(S.g_bits[w0]) : 0;
    const int c1 = w0 + 1 < n_words ? __popc(S.g_bits[w0 + 1]) : 0;
    int tot;
    const int ex = block_scan_excl(c0 + c1, S.g_scan, &tot);
    if (w0 < n_words) S.g_bpre[w0] = ex;
    if (w0 + 1 < n_words) S.g_bpre[w0 + 1] = ex + c0;
  }
  __syncthreads();
  // (4) each slot present: its rank d among the slots present, its rows
  for (int e = tid; e < kGroupTable; e += kDecThreads) {
    const int k = S.g_key[e];
    if (k >= 0) {
      const int d = S.g_bpre[k >> 5] + __popc(S.g_bits[k >> 5] & ((1u << (k & 31)) - 1u));
      int tot = 0;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) tot += S.g_cnt[e * kConsumerWarps + w];
      S.g_dtot[d] = tot;
      S.g_hd[e] = d;
    }
  }
  __syncthreads();
  // (5) first position and first item of each slot present (d < n_present)
  const int n_present = S.g_bpre[n_words - 1] + __popc(S.g_bits[n_words - 1]);
  int items_tot;
  {
    const int c = tid < n_present ? S.g_dtot[tid] : 0;
    int rows_tot;
    const int seg = block_scan_excl(c, S.g_scan, &rows_tot);
    const int it = block_scan_excl((c + kItemRows - 1) / kItemRows, S.g_scan, &items_tot);
    if (tid < n_present) {
      S.g_dseg[tid] = seg;
      S.g_ditem[tid] = it;
    }
  }
  __syncthreads();
  // (6) each row's grouped position; an item's first row records the item
  if (key >= 0) {
    const int d = S.g_hd[h];
    int before = 0;
    for (int w = 0; w < warp; ++w) before += S.g_cnt[h * kConsumerWarps + w];
    const int local = before + wrank;
    const int pos = S.g_dseg[d] + local;
    S.c_perm[pos] = tid;
    if (local % kItemRows == 0) {
      const int item = S.g_ditem[d] + local / kItemRows;
      S.c_item[item] = make_int4(key, pos, min(kItemRows, S.g_dtot[d] - local), 0);
      S.c_slot[item] = ld ? make_int4(rk, pa, pb, sc) : make_int4(0, -1, -1, 0);
    }
  }
  const int any_empty = __syncthreads_or(key >= 0 && !ld);
  if (blockIdx.x == 0 && tid == 0 && !any_bad && any_empty) set_status(a.status, LORA_ERR_NOT_LOADED);
  return items_tot;
}

// The plan path: the plan's items (up to kCacheItems), their slot records on
// the first target and the grouped rows (up to kCachePerm positions) copied
// into shared memory by all threads, the item count read alongside.
__device__ int plan_cache(const DecodeArgs &a, const DecSmem &S, int tid) {
  const int n_ci = min(a.items_cap, kCacheItems), n_cp = min(a.T, kCachePerm);
  int4 d = make_int4(0, 0, 0, 0);
  if (tid < n_ci) d = a.items[tid];
  for (int p = tid; p < n_cp; p += kDecThreads) S.c_perm[p] = a.perm[p];
  const int n_items = min(a.hdr[a.items_hdr], a.items_cap);
  if (tid < n_ci && tid < n_items) {
    const PoolView &p = a.pool;
    // (LORA_DEBUG: an item outside the pool's slots or the batch's rows is dropped)
    if (!dbg_ok(d.x >= 0 && d.x < p.n_slots && d.y >= 0 && d.z >= 0 && d.z <= kItemRows && d.y + d.z <= a.T,
                a.status))
      d = make_int4(0, 0, 0, 0);
    const int slot = d.x;
    const int rk = p.rank[(long long)slot * p.n_targets + a.tgt[0]];
    const int pa = block_page(p, slot, a.a_off[0], (long long)a.r_max * a.d_in * 2);
    const int pb = block_page(p, slot, a.bt_off[0], (long long)a.r_max * a.d_out * 2);
    const int sc = a.scales ? __float_as_int(a.scales[slot]) : 0;
    S.c_item[tid] = make_int4(d.x, d.y, d.z, 0);
    S.c_slot[tid] = make_int4(rk, pa, pb, sc);
  }
  __syncthreads();
  return n_items;
}

// ------------------------------------------------------------ the kernel
// Units of a launch: item-major, then target, then column range.  Column
// ranges per item: enough for about one unit per CTA of the launch, at most
// one per expand tile (a shrink-only launch has one unit per item and
// target).
template <int MODE>
struct UnitGeo {
  int nkt, nnt;  // tiles along d_in and d_out
  int nnu, npu;  // column ranges per item and target, expand tiles per range
  int total;

  __device__ UnitGeo(const DecodeArgs &a, int n_items) {
    nkt = (a.d_in / 8 + a.kcv - 1) / a.kcv;
    nnt = (a.d_out / 8 + a.kcv - 1) / a.kcv;
    const int per = max(n_items * a.n_tgt, 1);
    nnu = npu = 1;
    if (MODE != kShrinkOnly) {
      nnu = max(1, min((int)gridDim.x / per, nnt));
      npu = (nnt + nnu - 1) / nnu;
      nnu = (nnt + npu - 1) / npu;
    }
    total = n_items * a.n_tgt * nnu;
  }
};

// When a CTA of a launch that may prefetch early (DecodeArgs::early) last
// found no unit (%globaltimer, ns; one word per device, read by early_prefetch).
__device__ unsigned long long g_idle_ns;
__device__ __forceinline__ bool aborted(const DecSmem &S) { return *(volatile int *)S.misc != 0; }
__device__ __forceinline__ void set_abort(const DecSmem &S) { *(volatile int *)S.misc = 1; }

// Uneven column ranges (the copy warp; every CTA computes the same).  An
// item's expand tiles carry its rows of y in and out, so an item of many rows
// costs its CTA far more than a small one.  When the uniform split leaves
// SMs without a unit, each item of more than kSmallRows rows gets twice the
// uniform number of column ranges (at most one per expand tile), provided
// the units still fit one per SM; each of its units recomputes the item's
// shrink.  Returns the unit count (0: keep the uniform split) and writes the
// exclusive prefix of the items' range counts to S.c_pref.
constexpr int kSmallRows = 4;
__device__ int uneven_ranges(const DecodeArgs &a, const DecSmem &S, int n_items, int nnu, int nnt, int lane) {
  if (n_items > kCacheItems || (long long)n_items * nnu * a.n_tgt >= (long long)a.n_sms) return 0;
  const int big_k = min(2 * nnu, nnt);
  if (big_k == nnu) return 0;
  int base = 0;
  for (int t0 = 0; t0 < n_items; t0 += 32) {
    const int t = t0 + lane;
    const int k = t < n_items ? (S.c_item[t].z > kSmallRows ? big_k : nnu) : 0;
    int inc = k;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    if (t < n_items) S.c_pref[t] = base + inc - k;
    base += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (base == n_items * nnu || (long long)base * a.n_tgt > (long long)a.n_sms) return 0;  // nothing to gain
  if (lane == 0) S.c_pref[n_items] = base;
  __syncwarp();
  return base * a.n_tgt;
}

// Producer warp: walks the CTA's units (blockIdx.x, + gridDim.x, ...) and
// copies their tiles into the ring -- rows 0 .. r-1 of an adapter tile as one
// bulk copy (one contiguous range of the pool block), then one bulk copy per
// activation row.  Everything that does not change from tile to tile is set
// up once per unit, so a tile costs one header word, the expected bytes and
// the copies.
template <int MODE, int JB>
__device__ void produce(const DecodeArgs &a, const DecSmem &S, int n_items, int lane) {
  if (a.stall) return;  // (test of the bounded waits: the consumers' first wait runs out)
  const UnitGeo<MODE> U(a, n_items);
  const int NS = a.n_stages, NT = a.n_tgt;
  const bool fused = a.ids != nullptr;
  const int n_cached = fused ? n_items : min(n_items, kCacheItems);
  const int perm_cached = fused ? a.T : min(a.T, kCachePerm);
  const int act_base = a.r_max * a.kcv * 16;
  const long long tile_stride = (long long)a.r_max * a.kcv * 16;  // bytes between tiles of a block
  int stage = 0, fills = 0, rec = 0;
  uint32_t round = 0;  // completed passes over the ring (parity of the empty waits)
  // claims the next stage; false if waiting for it failed
  auto claim = [&]() -> bool {
    if (fills >= NS) {
      const bool ok = mbar_wait_bounded(&S.empty[stage], (round - 1) & 1, a.status, a.wait_ns);
      if (!ok) {
        set_abort(S);
        return false;
      }
      if (aborted(S)) return false;
    }
    return true;
  };
  auto advance = [&]() {
    ++fills;
    if (++stage == NS) {
      stage = 0;
      ++round;
    }
  };
  const int n_uneven = MODE == kFused ? uneven_ranges(a, S, n_items, U.nnu, U.nnt, lane) : 0;
  const int n_units = n_uneven > 0 ? n_uneven : U.total;
  if (a.early && (int)blockIdx.x >= n_units && lane == 0)
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(&g_idle_ns), "l"(global_ns()) : "memory");
  int item = blockIdx.x / (NT * U.nnu), rem = blockIdx.x - item * (NT * U.nnu);
  const int step_item = gridDim.x / (NT * U.nnu), step_rem = gridDim.x - step_item * (NT * U.nnu);
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    int ti, cur_item, e0, e1;
    if (n_uneven > 0) {
      // the item whose units hold u: the last t with NT * c_pref[t] <= u
      int lo_t = 0, hi_t = n_items - 1;
      while (lo_t < hi_t) {
        const int mid = (lo_t + hi_t + 1) >> 1;
        if (NT * S.c_pref[mid] <= u) lo_t = mid;
        else hi_t = mid - 1;
      }
      cur_item = lo_t;
      const int k = S.c_pref[lo_t + 1] - S.c_pref[lo_t];
      const int local = u - NT * S.c_pref[lo_t];
      ti = local / k;
      const int j = local - ti * k;
      e0 = j * U.nnt / k;
      e1 = (j + 1) * U.nnt / k;
    } else {
      ti = rem / U.nnu;
      const int nr = rem - ti * U.nnu;
      cur_item = item;
      item += step_item;
      rem += step_rem;
      if (rem >= NT * U.nnu) {
        rem -= NT * U.nnu;
        ++item;
      }
      e0 = nr * U.npu;
      e1 = MODE == kShrinkOnly ? e0 : min(e0 + U.npu, U.nnt);
    }
    // ---- the item and its slot on target ti
    int4 d;
    if (cur_item < n_cached) d = S.c_item[cur_item];
    else d = a.items[cur_item];
    if (!dbg_ok(d.x >= 0 && d.x < a.pool.n_slots && d.y >= 0 && d.z >= 0 && d.z <= kItemRows && d.y + d.z <= a.T,
                a.status))
      d = make_int4(0, 0, 0, 0);  // (LORA_DEBUG: dropped)
    const int slot = d.x, first = d.y, m = d.z;
    int r, page_a, page_b;
    float scale;
    if (cur_item < n_cached && ti == 0) {
      const int4 si = S.c_slot[cur_item];
      r = si.x;
      page_a = si.y;
      page_b = si.z;
      scale = __int_as_float(si.w);
    } else {
      const PoolView &p = a.pool;
      int val = 0;
      if (lane == 0) val = p.rank[(long long)slot * p.n_targets + a.tgt[ti]];
      if (lane == 1) val = block_page(p, slot, a.a_off[ti], (long long)a.r_max * a.d_in * 2);
      if (lane == 2) val = block_page(p, slot, a.bt_off[ti], (long long)a.r_max * a.d_out * 2);
      if (lane == 3) val = a.scales ? __float_as_int(a.scales[slot]) : 0;
      r = __shfl_sync(0xffffffffu, val, 0);
      page_a = __shfl_sync(0xffffffffu, val, 1);
      page_b = __shfl_sync(0xffffffffu, val, 2);
      scale = __int_as_float(__shfl_sync(0xffffffffu, val, 3));
    }
    if (r <= 0 || m <= 0) continue;  // nothing to add (a slot without this target)
    int myrow = lane < m ? (first + lane < perm_cached ? S.c_perm[first + lane] : a.perm[first + lane]) : 0;
    if (lane < m && !dbg_ok(myrow >= 0 && myrow < a.T, a.status)) myrow = -1;  // (LORA_DEBUG: not read or written)
    // lane L (1 <= L <= m) copies activation row L - 1: its x row and y row
    const int arow_raw = __shfl_sync(0xffffffffu, myrow, (lane + 31) & 31);
    const int arow = kDebugChecks && arow_raw < 0 ? 0 : arow_raw;
    const uint8_t *x_row = reinterpret_cast<const uint8_t *>(a.x + (long long)(arow / a.x_div) * a.ldx);
    const long long a_blk = S.tg[ti], b_blk = S.tg[kMaxMulti + ti], ycol = S.tg[2 * kMaxMulti + ti];
    const uint8_t *y_row = reinterpret_cast<const uint8_t *>(a.y + (long long)arow * a.ldy + ycol);
    // ---- the unit's record (its ring slot is free: every stage that named
    // it NS + 1 records ago has been released by now)
    UnitRec &R = S.rec[rec];
    if (lane == 0) {
      R.m = m;
      R.r = r;
      R.ycol = (int)ycol;
      R.scale = scale;
    }
    if (lane < kItemRows) R.rows[lane] = myrow;
    // ---- its tiles: the whole shrink, then the expand of column range nr
    const int ks = MODE == kExpandOnly ? U.nkt : 0;
    const int nvi = a.d_in / 8, nvo = a.d_out / 8;
    for (int t = ks; t < U.nkt + (e1 - e0); ++t) {
      const bool shrink = t < U.nkt;
      const int tt = shrink ? t : e0 + (t - U.nkt);  // tile index within its block
      if (!claim()) return;
      const int v_lo = tt * a.kcv;
      const int wv = min(a.kcv, (shrink ? nvi : nvo) - v_lo);
      const uint32_t row_bytes = (uint32_t)wv * 16u;
      uint8_t *buf = S.ring + stage * a.stage_bytes;
      __syncwarp();  // (the record's fields are written before the first stage names it)
      if (lane == 0) {
        const int first_t = shrink ? t == 0 : tt == e0;
        const int last_t = shrink ? t == U.nkt - 1 : tt == e1 - 1;
        S.hdr[stage] = StageHdr{(shrink ? kUnitShrink : kUnitExpand) | first_t << 4 | last_t << 5 | rec << 8, v_lo,
                                wv, 0};
        mbar_arrive_expect_tx(&S.full[stage], (uint32_t)(r + m) * row_bytes);
        // rows 0 .. r-1 of tile tt: one contiguous range of the block
        const long long off = (shrink ? a_blk : b_blk) + tt * tile_stride;
        const int page = shrink ? page_a : page_b;
        const uint32_t bytes = (uint32_t)r * row_bytes;
        if (page >= 0) {
          if (dbg_page_range(a.pool, page, off, bytes, a.status)) bulk_g2s(buf, page_addr(a.pool, page, off), bytes, &S.full[stage]);
          else bulk_g2s_redirect(buf, a.pool, bytes, &S.full[stage]);
        }
        else copy_pool_row(a.pool, slot, off, bytes, buf, &S.full[stage], a.status);
      }
      __syncwarp();  // (the expected bytes are registered before any copy can land)
      if (lane >= 1 && lane <= m)
        bulk_g2s(buf + act_base + (lane - 1) * a.pitch, (shrink ? x_row : y_row) + (long long)v_lo * 16, row_bytes,
                 &S.full[stage]);
      advance();
    }
    if (++rec == kRecs) rec = 0;
  }
  if (claim() && lane == 0) {
    S.hdr[stage] = StageHdr{kUnitEnd, 0, 0, 0};
    mbar_arrive_expect_tx(&S.full[stage], 0);
  }
}

// ------------------------------------------------------------ early prefetch
// Physical page of a slot's block as block_page() finds it, read from L2
// only (no line of the page table is left in L1 for later reads).
__device__ __forceinline__ int block_page_l2(const PoolView &p, int slot, long long first, long long bytes) {
  if (p.log2_page < 0) return __ldcg(p.pt + (long long)slot * p.pps);
  const long long pf = first >> p.log2_page, pl = (first + bytes - 1) >> p.log2_page;
  return pf == pl ? __ldcg(p.pt + (long long)slot * p.pps + pf) : -1;
}

// A launch on a plan may start before the kernel ahead of it on the stream
// has finished (programmatic dependent launch).  When that kernel is another
// such decode launch, the CTAs that start first are those that took an SM
// one of its CTAs without a unit gave back at once, and they would wait for
// it to finish anyway; so they bring the units' tiles and activation rows
// into L2 meanwhile: the first gridDim - n_units CTAs share the units (CTA
// b: units b, b + n_early, ...).  A CTA without a unit stamps g_idle_ns; a
// starting CTA counts itself early only if the stamp is under kEarlyNs old,
// so a launch that starts behind any other kernel (a base GEMM), or alone,
// skips all of this after one load.  The early CTAs read the plan and the
// pool's tables as they stand (L2-only loads, so nothing stale stays in L1),
// clamp every index into its buffer and use what they read for prefetch
// addresses only: a plan that is being rewritten, or a stamp left by a launch
// on another stream, costs a useless prefetch, never a wrong result.  All
// threads load, the copy warp prefetches.
constexpr unsigned long long kEarlyNs = 4000;
template <int MODE>
__device__ void early_prefetch(const DecodeArgs &a, const DecSmem &S, int tid) {
  const int lane = tid & 31, warp = tid >> 5, T = a.T;
  const PoolView &p = a.pool;
  if (tid == 0) {
    unsigned long long t;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(t) : "l"(&g_idle_ns) : "memory");
    S.misc[2] = global_ns() - t < kEarlyNs;
  }
  __syncthreads();
  if (!S.misc[2]) return;
  const int n_ci = min(a.items_cap, kCacheItems);
  if (tid < n_ci) {
    const int4 d = __ldcg(a.items + tid);
    const int slot = min(max(d.x, 0), p.n_slots - 1), first = min(max(d.y, 0), T);
    S.c_item[tid] = make_int4(slot, first, min(max(d.z, 0), min(kItemRows, T - first)), 0);
  }
  for (int q = tid; q < T; q += kDecThreads) S.c_perm[q] = min(max(__ldcg(a.perm + q), 0), T - 1);
  __syncthreads();
  if (warp == kProdWarp) {
    int n_items = lane == 0 ? __ldcg(a.hdr + a.items_hdr) : 0;
    n_items = min(max(__shfl_sync(0xffffffffu, n_items, 0), 0), n_ci);
    const UnitGeo<MODE> U(a, n_items);
    const int NT = a.n_tgt;
    const int n_uneven = MODE == kFused ? uneven_ranges(a, S, n_items, U.nnu, U.nnt, lane) : 0;
    const int n_units = n_uneven > 0 ? n_uneven : U.total;
    const int n_early = (int)gridDim.x - n_units;
    const int nvi = a.d_in / 8, nvo = a.d_out / 8;
    const long long tile_stride = (long long)a.r_max * a.kcv * 16;
    for (int u0 = blockIdx.x; u0 < n_units && (int)blockIdx.x < n_early; u0 += 32 * n_early) {
      // lane j: where unit u0 + j * n_early lies and its slot's record
      const int u = u0 + lane * n_early;
      int it = 0, ti = 0, e0 = 0, e1 = 0, r = 0, pa = -1, pb = -1;
      if (u < n_units) {
        if (n_uneven > 0) {
          int lo_t = 0, hi_t = n_items - 1;
          while (lo_t < hi_t) {
            const int mid = (lo_t + hi_t + 1) >> 1;
            if (NT * S.c_pref[mid] <= u) lo_t = mid;
            else hi_t = mid - 1;
          }
          it = lo_t;
          const int k = S.c_pref[lo_t + 1] - S.c_pref[lo_t];
          const int local = u - NT * S.c_pref[lo_t];
          ti = local / k;
          const int j = local - ti * k;
          e0 = j * U.nnt / k;
          e1 = (j + 1) * U.nnt / k;
        } else {
          it = u / (NT * U.nnu);
          const int rem = u - it * (NT * U.nnu);
          ti = rem / U.nnu;
          e0 = (rem - ti * U.nnu) * U.npu;
          e1 = MODE == kShrinkOnly ? e0 : min(e0 + U.npu, U.nnt);
        }
        const int slot = S.c_item[it].x;
        r = min(max(__ldcg(p.rank + (long long)slot * p.n_targets + a.tgt[ti]), 0), a.r_max);
        pa = block_page_l2(p, slot, a.a_off[ti], (long long)a.r_max * a.d_in * 2);
        pb = block_page_l2(p, slot, a.bt_off[ti], (long long)a.r_max * a.d_out * 2);
      }
      const int nu = min(32, (n_units - u0 + n_early - 1) / n_early);
      for (int j = 0; j < nu; ++j) {
        const int uit = __shfl_sync(0xffffffffu, it, j), uti = __shfl_sync(0xffffffffu, ti, j);
        const int ue0 = __shfl_sync(0xffffffffu, e0, j), ue1 = __shfl_sync(0xffffffffu, e1, j);
        const int ur = __shfl_sync(0xffffffffu, r, j);
        const int upa = __shfl_sync(0xffffffffu, pa, j), upb = __shfl_sync(0xffffffffu, pb, j);
        const int4 d = S.c_item[uit];
        if (ur == 0 || d.z == 0) continue;
        for (int q = lane; q < U.nkt + (ue1 - ue0); q += 32) {  // adapter rows, one tile per lane
          const bool sq = q < U.nkt;
          const int tq = sq ? q : ue0 + (q - U.nkt);
          const int page = sq ? upa : upb;
          const long long off = (sq ? a.a_off[uti] : a.bt_off[uti]) + tq * tile_stride;
          if (page >= 0 && page < p.n_pages)
            bulk_prefetch_l2(page_addr(p, page, off),
                             (uint32_t)ur * (uint32_t)min(a.kcv, (sq ? nvi : nvo) - tq * a.kcv) * 16u);
        }
        if (lane < d.z) {  // the item's x rows and its y rows in the unit's columns
          const int row = S.c_perm[d.y + lane];
          bulk_prefetch_l2(a.x + (long long)(row / a.x_div) * a.ldx, (uint32_t)nvi * 16u);
          const int v0 = ue0 * a.kcv, v1 = min(ue1 * a.kcv, nvo);
          if (v1 > v0) bulk_prefetch_l2(a.y + (long long)row * a.ldy + a.y_col[uti] + (long long)v0 * 8, (uint32_t)(v1 - v0) * 16u);
        }
      }
    }
  }
  __syncthreads();  // (the shared arrays are rewritten from the plan next)
}

// Consumer warps: the contractions, out of the ring.
template <int MODE, int JB>
__device__ void consume(const DecodeArgs &a, const DecSmem &S, int tid) {
  const int lane = tid & 31, warp = tid >> 5;
  const int NS = a.n_stages, pitch = a.pitch;
  const int act_base = a.r_max * a.kcv * 16;  // activation rows follow the adapter tile
  int stage = 0;
  uint32_t phase = 0;
  // Waits for the current stage; false once the producer is done (or a wait
  // gave up: the abort flag is then set).
  auto acquire = [&]() -> bool {
    const bool got = cons_sync_and(mbar_wait_bounded(&S.full[stage], phase, a.status, a.wait_ns));
    if (!got) {
      if (tid == 0) set_abort(S);
      return false;
    }
    return (S.hdr[stage].bits & 15) != kUnitEnd;
  };
  // An expand stage goes back to the producer only once the bulk copies of
  // its y rows have read it; with three or more stages this warp hands it
  // back after its next tile (pend), so that the copies run during that tile.
  int pend = -1;
  auto release = [&]() {
    __syncwarp();
    if (lane == 0) {
      if (pend >= 0) {
        bulk_wait_read();
        mbar_arrive(&S.empty[pend]);
      }
      mbar_arrive(&S.empty[stage]);  // this warp is done with the stage
    }
    pend = -1;
    if (++stage == NS) {
      stage = 0;
      phase ^= 1u;
    }
  };
  auto release_after_copies = [&]() {
    if (NS < 3) {  // a two-stage ring: holding one back would stall the producer
      if (lane == 0) bulk_wait_read();
      release();
      return;
    }
    __syncwarp();
    if (lane == 0 && pend >= 0) {
      bulk_wait_read_but_newest();  // (the previous expand stage's copies, not this one's)
      mbar_arrive(&S.empty[pend]);
    }
    pend = stage;
    if (++stage == NS) {
      stage = 0;
      phase ^= 1u;
    }
  };
  while (acquire()) {
    StageHdr H = S.hdr[stage];
    if ((H.bits & 15) == kUnitShrink) {
      // the unit's shrink tiles, this one up to the one marked last; the
      // accumulator lives only here
      float sacc[JB < 2 ? 2 : JB][4];  // this warp's MMA fragment of the unit's V so far
#pragma unroll
      for (int nt = 0; nt < (JB < 2 ? 2 : JB); ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
      while (true) {
        const bool last = (H.bits >> 5) & 1;
        const UnitRec &R = S.rec[H.bits >> 8];
        const int m = R.m, r = R.r, wv = H.wv;
        uint8_t *buf = S.ring + stage * a.stage_bytes;
        const uint32_t buf_u = smem_u32(buf);
        if (wv == full_tile_chunks(JB))
          shrink_full<JB, full_tile_chunks(JB) / 2 / kConsumerWarps>(buf_u, buf_u + act_base, pitch, wv, r, m, sacc,
                                                                       lane, warp);
        else
          shrink_mma<JB>(buf_u, buf_u + act_base, pitch, wv, r, m, sacc, lane, warp);
        if (last) {
          // v of the unit's rows: the warps' fragments meet in the stage's
          // adapter rows and are summed in fixed warp order
          cons_sync();
          float *red = reinterpret_cast<float *>(buf);
          const int n = m * r;
          shrink_spill<JB>(sacc, r, m, red + warp * kItemRows * r, lane);
          fence_proxy_async_smem();
          cons_sync();
          if (MODE == kShrinkOnly) {  // to the caller: ranks r .. r_max-1 as zeros
            for (int e = tid; e < m * a.r_max; e += kConsumerThreads) {
              const int i = e / a.r_max, j = e - i * a.r_max;
              float s = 0.f;
              if (j < r) {
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) s += red[w * kItemRows * r + i * r + j];
              }
              if (!kDebugChecks || R.rows[i] >= 0) a.v[(long long)R.rows[i] * a.ldv + j] = s;
            }
          } else {
            for (int e = tid; e < n; e += kConsumerThreads) {
              float s = 0.f;
#pragma unroll
              for (int w = 0; w < kConsumerWarps; ++w) s += red[w * kItemRows * r + e];
              const int i = e / r, j = e - i * r;
              S.v[i * a.r_max + j] = s;
            }
          }
          release();
          break;
        }
        release();
        if (!acquire()) goto done;
        H = S.hdr[stage];
      }
    } else {
      const bool first = (H.bits >> 4) & 1;
      const UnitRec &R = S.rec[H.bits >> 8];
      const int m = R.m, r = R.r, wv = H.wv, v_lo = H.v_lo;
      uint8_t *buf = S.ring + stage * a.stage_bytes;
      const uint32_t buf_u = smem_u32(buf);
      if (MODE == kExpandOnly && first) {  // the caller's v
        for (int e = tid; e < m * r; e += kConsumerThreads) {
          const int i = e / r, j = e - i * r;
          S.v[i * a.r_max + j] = (!kDebugChecks || R.rows[i] >= 0) ? a.v[(long long)R.rows[i] * a.ldv + j] : 0.f;
        }
      }
      cons_sync();  // S.v complete (written by the shrink's last tile or just above)
      ExpandA<JB> va;  // the unit's V as MMA operand fragments (hi + lo)
      expand_prepare<JB>(S.v, a.r_max, r, m, va, lane);
      uint8_t *yb = buf + act_base;
      expand_mma<JB>(buf_u, yb, smem_u32(S.zero), pitch, wv, r, m, va, R.scale, lane, warp);
      // the updated rows out (warp w: rows w, w + 8).  A few rows: the
      // warp's lanes store consecutive 16-byte chunks (whole lines per
      // instruction) and the stage goes back at once.  More: one bulk copy
      // per row, the stage handed back once the copies have read it.
      if (m <= kStoreRowsMax) {
        cons_sync();
        for (int i = warp; i < m; i += kConsumerWarps) {
          if (kDebugChecks && R.rows[i] < 0) continue;  // (LORA_DEBUG: a row that failed its check)
          const uint8_t *src = yb + i * pitch;
          uint16_t *dst = a.y + (long long)R.rows[i] * a.ldy + R.ycol + (long long)v_lo * 8;
          for (int ch = lane; ch < wv; ch += 32)
            *reinterpret_cast<uint4 *>(dst + ch * 8) = *reinterpret_cast<const uint4 *>(src + ch * 16);
        }
        release();
      } else {
        fence_proxy_async_smem();
        cons_sync();
        if (lane == 0) {
          const long long col = R.ycol + (long long)v_lo * 8;
          if (warp < m && (!kDebugChecks || R.rows[warp] >= 0))
            bulk_s2g(a.y + (long long)R.rows[warp] * a.ldy + col, yb + warp * pitch, (uint32_t)wv * 16u);
          if (warp + 8 < m && (!kDebugChecks || R.rows[warp + 8] >= 0))
            bulk_s2g(a.y + (long long)R.rows[warp + 8] * a.ldy + col, yb + (warp + 8) * pitch, (uint32_t)wv * 16u);
          bulk_commit();
        }
        release_after_copies();
      }
    }
  }
done:
  if (lane == 0) bulk_wait_all();  // this warp's y rows are in global memory
}

template <int MODE, int JB>
__global__ void __launch_bounds__(kDecThreads, dec_min_blocks(JB)) decode_kernel(const __grid_constant__ DecodeArgs a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(128) uint8_t smem[];
  const DecSmem S = dec_carve(smem, a);
  if (tid == 0) {
    for (int s = 0; s < a.n_stages; ++s) {
      mbar_init(&S.full[s], 1);                // the producer (with the stage's bytes)
      mbar_init(&S.empty[s], kConsumerWarps);  // every consumer warp, once done with the stage
    }
    *S.misc = 0;
    fence_mbar_init();
  }
  if (tid < 16) reinterpret_cast<uint32_t *>(S.zero)[tid] = 0u;
  if (tid < kMaxMulti) {  // (kernel parameters: read while the previous launch may still run)
    S.tg[tid] = a.a_off[tid];
    S.tg[kMaxMulti + tid] = a.bt_off[tid];
    S.tg[2 * kMaxMulti + tid] = a.y_col[tid];
  }
  __syncthreads();
  if (a.early && !a.stall) early_prefetch<MODE>(a, S, tid);
  griddep_wait();
  griddep_launch_dependents();
  const int n_items = a.ids ? fused_group(a, S, tid) : plan_cache(a, S, tid);  // every thread
  if (warp == kProdWarp) produce<MODE, JB>(a, S, n_items, lane);
  else consume<MODE, JB>(a, S, tid);
}

// ------------------------------------------------------------ host side
struct DecodeGeo {
  int kcv, pitch, stage_bytes, n_stages, smem;
};

// Ring geometry for a slot rank: the pool's tiles and as many stages (2 ..
// kMaxStages) as fit in about 113 KB, so that two CTAs share an SM; where
// two stages do not fit in that (rank 16 and below: 1024-column tiles), one
// CTA per SM with up to 210 KB of stages.
static DecodeGeo decode_geometry(int r_max) {
  DecodeGeo g;
  g.kcv = pool_tile_cols(r_max) / 8;
  g.pitch = g.kcv * 16 + 16;
  g.stage_bytes = r_max * g.kcv * 16 + kItemRows * g.pitch;
  const int extra = dec_extra_bytes(r_max);
  const int budget = (2 * std::max(g.stage_bytes, kRingMin / 2) + extra <= 113 * 1024) ? 113 * 1024 : 210 * 1024;
  g.n_stages = 2;
  for (int ns = kMaxStages; ns > 2; --ns)
    if (std::max(ns * g.stage_bytes, kRingMin) + extra <= budget) {
      g.n_stages = ns;
      break;
    }
  g.smem = std::max(g.n_stages * g.stage_bytes, kRingMin) + extra;
  return g;
}

// Rank rows per warp of the shrink: the smallest power of two with
// 8 * JB >= r_max (ranks below r_max use the same kernel).
static int jb_for(int r_max) { return r_max <= 8 ? 1 : r_max <= 16 ? 2 : r_max <= 32 ? 4 : 8; }

template <int MODE, int JB>
static cudaError_t launch_one(const DecodeArgs &a, int grid, int smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<MODE, JB>, a);
}

template <int MODE>
static cudaError_t launch_mode(const DecodeArgs &a, int jb, int grid, int smem, cudaStream_t st) {
  switch (jb) {
    case 1: return launch_one<MODE, 1>(a, grid, smem, st);
    case 2: return launch_one<MODE, 2>(a, grid, smem, st);
    case 4: return launch_one<MODE, 4>(a, grid, smem, st);
    default: return launch_one<MODE, 8>(a, grid, smem, st);
  }
}

template <int MODE, int JB>
static cudaError_t set_attrs(int bytes) {
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<MODE, JB>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_kernel<MODE, JB>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  return e;
}

template <int MODE>
static cudaError_t set_attrs_all(int bytes) {
  cudaError_t e = set_attrs<MODE, 1>(bytes);
  if (e == cudaSuccess) e = set_attrs<MODE, 2>(bytes);
  if (e == cudaSuccess) e = set_attrs<MODE, 4>(bytes);
  if (e == cudaSuccess) e = set_attrs<MODE, 8>(bytes);
  return e;
}

template <int JB>
static cudaError_t per_sm(int *n, int smem) {
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, decode_kernel<kFused, JB>, kDecThreads, smem);
}

static std::atomic<unsigned long long> g_wait_ns{kSpinNs};

void set_wait_limit_ns(unsigned long long ns) { g_wait_ns.store(ns == 0 ? kSpinNs : ns); }
unsigned long long wait_limit_ns() { return g_wait_ns.load(); }

int decode_setup(lora_pool *pool) {
  // The attribute is per function: set it to what the largest geometry
  // needs, so that pools of different r_max can coexist.
  int smem_cap = 0;
  for (int r = 1; r <= kRMax; ++r) smem_cap = std::max(smem_cap, decode_geometry(r).smem);
  if (set_attrs_all<kFused>(smem_cap) != cudaSuccess || set_attrs_all<kShrinkOnly>(smem_cap) != cudaSuccess ||
      set_attrs_all<kExpandOnly>(smem_cap) != cudaSuccess)
    return LORA_ERR_CUDA;
  const DecodeGeo g = decode_geometry(pool->r_max);
  int n = 0;
  cudaError_t e;
  switch (jb_for(pool->r_max)) {
    case 1: e = per_sm<1>(&n, g.smem); break;
    case 2: e = per_sm<2>(&n, g.smem); break;
    case 4: e = per_sm<4>(&n, g.smem); break;
    default: e = per_sm<8>(&n, g.smem); break;
  }
  int sms = 0;
  if (e != cudaSuccess || n < 1 ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, pool->device) != cudaSuccess || sms < 1) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  pool->decode_per_sm = n;
  pool->decode_max_ctas = n * sms;
  return LORA_OK;
}

int launch_decode(lora_pool *pool, const DecodeCall &c, cudaStream_t st) {
  if (c.n_tgt < 1 || c.n_tgt > kMaxMulti || c.T < 1) return LORA_ERR_INVALID_ARG;
  if (c.ids ? c.T > kFusedMaxT : c.ws == nullptr) return LORA_ERR_INVALID_ARG;
  DecodeArgs a;
  a.pool = pool->view();
  a.d_in = pool->targets[c.targets[0]].d_in;
  a.d_out = pool->targets[c.targets[0]].d_out;
  a.r_max = pool->r_max;
  a.n_tgt = c.n_tgt;
  for (int i = 0; i < kMaxMulti; ++i) {
    const int t = c.targets[i < c.n_tgt ? i : 0];
    a.tgt[i] = t;
    a.a_off[i] = pool->a_off[t];
    a.bt_off[i] = pool->bt_off[t];
    a.y_col[i] = (c.y_cols && i < c.n_tgt) ? c.y_cols[i] : 0;
  }
  a.x = static_cast<const uint16_t *>(c.x);
  a.ldx = c.ldx;
  a.y = static_cast<uint16_t *>(c.y);
  a.ldy = c.ldy;
  a.scales = c.scales;
  const PlanLayout L = plan_layout(c.T);
  a.early = !c.ids && c.mode != kExpandOnly && c.T <= kCachePerm;
  if (c.ids) {
    a.hdr = nullptr;
    a.perm = nullptr;
    a.items = nullptr;
  } else {
    const PlanView pv = plan_view(c.ws, L);
    a.hdr = pv.hdr;
    a.perm = pv.perm;
    a.items = pv.items;
  }
  a.items_hdr = c.items_hdr;
  a.items_cap = L.i_max;
  a.ids = c.ids;
  a.T = c.T;
  a.x_div = c.x_div;
  a.moe_topk = c.moe_topk;
  a.moe_k = c.moe_k;
  a.moe_e = c.moe_e;
  a.v = c.v;
  a.ldv = c.ldv;
  a.n_sms = pool->decode_max_ctas / std::max(pool->decode_per_sm, 1);
  a.stall = c.stall;
  a.status = pool->d_status;
  a.wait_ns = g_wait_ns.load();
  const DecodeGeo g = decode_geometry(pool->r_max);
  a.kcv = g.kcv;
  a.pitch = g.pitch;
  a.stage_bytes = g.stage_bytes;
  a.n_stages = g.n_stages;
  // One wave of CTAs; no more CTAs than the units a batch of this size can
  // produce (items x targets x expand tiles).
  const long long items = c.ids ? (long long)std::min(c.T, pool->n_slots) + (c.T + kItemRows - 1) / kItemRows
                                : (long long)L.i_max;
  const long long nnt = (a.d_out / 8 + g.kcv - 1) / g.kcv;
  const long long units = items * c.n_tgt * (c.mode == kShrinkOnly ? 1 : nnt);
  const int grid = (int)std::max<long long>(1, std::min<long long>(units, pool->decode_max_ctas));
  const int jb = jb_for(pool->r_max);
  g_launches.fetch_add(1);
  cudaError_t e;
  if (c.mode == kFused) e = launch_mode<kFused>(a, jb, grid, g.smem, st);
  else if (c.mode == kShrinkOnly) e = launch_mode<kShrinkOnly>(a, jb, grid, g.smem, st);
  else e = launch_mode<kExpandOnly>(a, jb, grid, g.smem, st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

}  // namespace lora
