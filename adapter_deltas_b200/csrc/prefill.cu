// prefill.cu -- tensor-core path of the multi-LoRA delta for long segments.
//
// A prefill batch arrives as contiguous segments of rows that share an
// adapter.  A segment long enough is a real dense contraction, so its rows go
// through the 5th-generation tensor cores in tiles of 128 rows:
//     V = X A_a^T          (shrink: M=128 rows, N=rank, K=d_in)
//     Y += s_a * V B_a^T   (expand: M=128 rows, N=d_out, K=rank)
// the per-request term of y = xW + (x A_i) B_i (alpha / r) ("Multi-LoRA
// Serving: Why 100 Adapters Fit on One GPU", section "Why can't you just merge
// LoRA weights into the base model?"); the same page (section "How does one
// batch run 30 different adapters at once?") notes that the delta is a small
// cost against a 4096-token prefill -- it is bound by the bytes of x and y.
//
// B200 mapping: two launches, each a flat list of equal work units spread
// over all SMs, so that no SM waits on another's tile.
//   shrink  unit = (tile, k-slice of d_in): TMA streams the slice's x blocks
//           (2-D tiled, 128-byte swizzle, no multicast) through a stage ring
//           fed by a producer warp; an MMA warp accumulates X_slice A_slice^T
//           in TMEM (tcgen05.mma kind::f16, bf16 in, fp32 accumulate); the
//           epilogue warps write the fp32 partial V of the tile's own rows to
//           the workspace.
//   expand  unit = (tile, 256 columns of d_out): the partials of the tile's
//           rows are summed in fixed k-slice order (deterministic), split
//           into two bf16 terms (hi + lo, about 16 bits of V kept), and
//           multiplied by the B^T columns in TMEM; the epilogue adds s * acc
//           to y (fetched by TMA) in fp32 and stores bf16 for the tile's own
//           rows, 8 lanes per 128-byte row.
// The shrink's A slice arrives by one bulk copy per rank row (through the
// page table, pieces at page boundaries) into a row-major staging area and is
// moved into the MMA layout in shared memory; the expand's B^T columns come
// by 16-byte cp.async, one page lookup per row.  Every wait is bounded.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "internal.cuh"
#include "tc.cuh"

namespace lora {

constexpr int kBoxCols = 64;                 // TMA box: 64 bf16 (128 B) x 128 rows
constexpr int kBoxBytes = kBoxCols * 2 * kMmaRows;
constexpr int kChunkCols = 128;              // expand MMA N
constexpr int kPfRankCap = 32;
constexpr int kSms = 148;                       // B200 SM count (grid sizing heuristics only)
// shrink kernel
constexpr int kShEpiWarps = 4;
constexpr int kShEpiThreads = 32 * kShEpiWarps;
constexpr int kShThreads = kShEpiThreads + 64;   // + TMA producer warp + MMA warp
constexpr int kShMaxStages = 8;
constexpr int kShMaxBlocks = 16;                  // x blocks (64 columns) per k-slice
constexpr int kShTmemCols = 32;
// expand kernel
constexpr int kExThreads = 128;                   // warp w: tile rows 32w .. 32w + 31
constexpr int kGroupCols = kChunkCols;            // d_out columns per unit (one MMA chunk, two y boxes)
constexpr int kGroupBoxes = kGroupCols / kBoxCols;
constexpr int kExTmemCols = kChunkCols;
constexpr int kExMaxPerSm = 4;                    // 4 x 128 TMEM columns = the SM's 512
constexpr int kSmemPerSm = 228 * 1024;            // shared memory per SM (each CTA also takes 1 KB)

struct __align__(64) PrefillArgs {
  CUtensorMap tmap_x;   // x [T, d_in], box 64 x 128, 128-byte swizzle
  CUtensorMap tmap_y;   // y [T, d_out], same box
  PoolView pool;
  int target, d_in, d_out, T;
  long long a_off, bt_off;
  uint16_t *y;
  long long ldy;
  const float *scales;
  const int32_t *hdr;
  const int4 *tiles;
  int *status;
  float *vpart;         // [n_ks][T][r_cap] fp32 partial V of each k-slice
  int r_cap;            // 16 or 32
  int pool_r_max;       // rank rows of a slot's blocks (<= r_cap)
  int kb_per;           // x blocks per k-slice
  int n_ks;             // k-slices
  int n_stages;         // shrink ring stages
  int n_groups;         // expand column groups
};

// Address of the 16-byte chunk at logical byte `off` of a slot's block: on
// the block's page when it has one (page >= 0), else through the page table.
__device__ __forceinline__ const uint8_t *block_chunk(const PoolView &pool, int slot, int page, long long off,
                                                      int *status) {
  if (page >= 0) return dbg_page_range(pool, page, off, 16, status) ? page_addr(pool, page, off) : pool.base;
  if (!dbg_slot_range(pool, slot, off, 16, status)) return pool.base;  // (LORA_DEBUG: redirected)
  long long room;
  const uint8_t *src = pool_addr(pool, slot, off, &room);
  if (!src) {
    set_status(status, LORA_ERR_NOT_LOADED);
    src = pool.base;
  }
  return src;
}

// ============================================================ shrink kernel
struct ShSmem {
  uint8_t *ring, *aw, *stg;  // x stages; A slice in the MMA layout; A slice rows as copied
  uint64_t *full, *empty, *w_full, *a_land, *sh_done, *stg_free;
  uint32_t *tmem_slot;
};

__host__ __device__ inline int sh_smem_bytes(int n_stages, int r_cap, int kb_per) {
  return 1024 /* alignment slack */ + n_stages * kBoxBytes + 2 * r_cap * kb_per * kBoxCols * 2 +
         (2 * kShMaxStages + 4) * 8 + 16;
}

// Warp roles: warps 0-3 copy the adapter slice and write the partial V (warp
// w owns TMEM lanes / tile rows 32w .. 32w + 31); warp 4 issues the TMA
// loads; warp 5 issues the MMAs.  Every role walks the same unit list.
__global__ void __launch_bounds__(kShThreads, 1) pf_shrink_kernel(const __grid_constant__ PrefillArgs a) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NS = a.n_stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ShSmem S;
  {
    uint8_t *p = base;
    S.ring = p; p += NS * kBoxBytes;
    S.aw = p; p += a.r_cap * a.kb_per * kBoxCols * 2;
    S.stg = p; p += a.r_cap * a.kb_per * kBoxCols * 2;
    uint64_t *b = reinterpret_cast<uint64_t *>(p);
    S.full = b; b += kShMaxStages;
    S.empty = b; b += kShMaxStages;
    S.w_full = b++;
    S.a_land = b++;
    S.sh_done = b++;
    S.stg_free = b++;
    S.tmem_slot = reinterpret_cast<uint32_t *>(b);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(S.tmem_slot)),
                 "r"(kShTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == kShEpiThreads) {
    for (int i = 0; i < kShMaxStages; ++i) {
      mbar_init(&S.full[i], 1);
      mbar_init(&S.empty[i], 1);
    }
    mbar_init(S.w_full, kShEpiThreads);
    mbar_init(S.a_land, 1);
    mbar_init(S.sh_done, 1);
    mbar_init(S.stg_free, 1);
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_x)) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *S.tmem_slot;
  griddep_wait();
  griddep_launch_dependents();  // the expand may start its y and B^T loads

  bool alive = true;
  const int n_units = a.hdr[kHdrTiles] * a.n_ks;
  const int nkb_all = (a.d_in + kBoxCols - 1) / kBoxCols;
  const uint32_t lbo_a = (uint32_t)(a.r_cap / 8) * 128u;  // k-group stride of the A_a slice
  const uint32_t aw_u = smem_u32(S.aw), ring_u = smem_u32(S.ring);
  uint32_t gbase = 0;   // ring uses so far: use g sits in stage g % NS with phase (g / NS) & 1
  uint32_t ucount = 0;  // units multiplied so far (w_full / sh_done phases)
  uint32_t ucopy = 0;   // units whose A slice was copied (a_land phases; stg_free phases: ucopy - 1)

  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    const int tile = u / a.n_ks, ks = u - tile * a.n_ks;
    const int kb0 = ks * a.kb_per, nkb = min(a.kb_per, nkb_all - kb0);
    if (nkb <= 0) continue;
    const int4 d = a.tiles[tile];
    // (LORA_DEBUG: a tile outside the pool's slots or the batch's rows is skipped by every role)
    if (!dbg_ok(d.x >= 0 && d.x < a.pool.n_slots && d.y >= 0 && d.z > 0 && d.z <= kMmaRows && d.y + d.z <= a.T,
                a.status))
      continue;
    const int slot = d.x, row0 = d.y, m = d.z;

    // The A slice does not wait for the rank: all r_cap rows come (the pool
    // keeps an adapter's rows past its rank at zero), so the copies leave as
    // soon as the tile record is known.
    // The slice is whole pool tiles (k-slices start on tile boundaries): the
    // first rows_cp rows of each tile are one contiguous range of the block,
    // copied as they are (tile after tile, tile stride r_cap rows).
    const int cols = min(nkb * kBoxCols, a.d_in - kb0 * kBoxCols);
    const int tc = pool_tile_cols(a.pool_r_max), tcc = tc / 8;
    const int tile0 = kb0 * kBoxCols / tc, n_tl = (cols + tc - 1) / tc;
    const int rows_cp = min(a.r_cap, a.pool_r_max);

    if (warp == kShEpiWarps) {
      // ------------------------------------------------ TMA producer
      // The A slice first (the MMAs wait for it; issued behind this CTA's
      // x boxes it would queue behind every CTA's first wave of x), once the
      // epilogue is done with the previous unit's staged slice; then the x
      // boxes (x depends only on the tile record; a unit whose adapter turns
      // out absent still passes its blocks through the ring, the MMA warp
      // just does not multiply them).
      if (ucopy > 0) warp_wait(S.stg_free, (ucopy - 1) & 1u, a.status, alive);
      if (lane == 0) mbar_arrive_expect_tx(S.a_land, (uint32_t)rows_cp * (uint32_t)cols * 2u);
      __syncwarp();
      if (lane < n_tl && alive) {
        const int t = tile0 + lane;
        const int tw = min(tcc, a.d_in / 8 - t * tcc);
        copy_pool_row(a.pool, slot, a.a_off + (long long)t * a.pool_r_max * tcc * 16, (uint32_t)(rows_cp * tw * 16),
                      S.stg + lane * a.r_cap * tcc * 16, S.a_land, a.status);
      }
      __syncwarp();
      if (lane == 0) {
        for (int i = 0; i < nkb; ++i) {
          const uint32_t g = gbase + i, st = g % NS;
          if (g >= (uint32_t)NS && !pf_wait(&S.empty[st], ((g / NS) - 1) & 1, a.status, alive)) break;
          mbar_arrive_expect_tx(&S.full[st], kBoxBytes);
          tma_load_2d(S.ring + st * kBoxBytes, &a.tmap_x, (kb0 + i) * kBoxCols, row0, &S.full[st]);
        }
      }
      __syncwarp();
      gbase += nkb;
      ++ucopy;
      continue;
    }
    const int r = a.pool.rank[slot * a.pool.n_targets + a.target];
    const bool use = r > 0 && r <= a.r_cap;
    if (r > a.r_cap && tid == 0) set_status(a.status, LORA_ERR_INVALID_ARG);
    const int R = (r + 15) & ~15;
    const uint32_t par = ucount & 1u;

    if (warp == kShEpiWarps + 1) {
      // ------------------------------------------------ MMA issuer
      if (lane == 0) {
        if (use) pf_wait(S.w_full, par, a.status, alive);
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(use ? R : 16, false);
        for (int i = 0; i < nkb; ++i) {
          const uint32_t g = gbase + i, st = g % NS;
          pf_wait(&S.full[st], (g / NS) & 1, a.status, alive);
          tc_fence_after();
          const uint32_t xa = ring_u + st * kBoxBytes;
#pragma unroll
          for (int kk = 0; kk < kBoxCols / 16; ++kk) {
            const uint64_t ad = smem_desc(xa + kk * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(aw_u + (uint32_t)(i * 4 + kk) * 2 * lbo_a, lbo_a, 128, 0);
            if (alive && use) mma_bf16(tmem, ad, bd, idesc, (i | kk) != 0);
          }
          mma_commit(&S.empty[st]);  // the stage is free once these MMAs have read it
        }
        if (use) mma_commit(S.sh_done);
      }
      __syncwarp();
    } else {
      // ------------------------------------------------ epilogue warps
      // (1) the k-slice of A_a, copied above in the pool's tiled arrangement
      // (one bulk copy per tile), moved into the MMA's K-major core-matrix
      // layout: 8 rank rows x 4 chunks per warp access, so each 128-byte core
      // matrix is written whole; zero rows from r up to R and zero columns
      // beyond d_in
      warp_wait(S.a_land, ucopy & 1u, a.status, alive);
      if (use) {
        const int kv_n = nkb * (kBoxCols / 8);
        const int jl = lane & 7, vo = lane >> 3;
        const int tsh = 31 - __clz(tcc);  // (tcc is a power of two)
        for (int jg = 0; jg < R / 8; ++jg) {
          const int j = jg * 8 + jl;
          for (int kv = warp * 4 + vo; kv < kv_n; kv += kShEpiWarps * 4) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (j < r && kv * 8 < cols) {
              const int tl = kv >> tsh, c = kv & (tcc - 1);
              const int tw = min(tcc, a.d_in / 8 - (tile0 + tl) * tcc);
              v = *reinterpret_cast<const uint4 *>(S.stg + (tl * a.r_cap * tcc + j * tw + swz_chunk(c, j, tw)) * 16);
            }
            *reinterpret_cast<uint4 *>(S.aw + kv * lbo_a + jg * 128 + jl * 16) = v;
          }
        }
      }
    }
    if (use && warp < kShEpiWarps) {
      fence_async_smem();  // generic-proxy writes -> visible to the MMAs (async proxy)
      tc_fence_before();   // the previous unit's TMEM reads are done
      pf_arrive(S.w_full);

      // (2) the partial V of row tid of the tile -> workspace
      warp_wait(S.sh_done, par, a.status, alive);
      tc_fence_after();
      if (alive) {
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float v[kPfRankCap];
        tmem_ld16(lane_base, *reinterpret_cast<float(*)[16]>(v));
        if (R > 16) tmem_ld16(lane_base + 16, *reinterpret_cast<float(*)[16]>(v + 16));
        tmem_wait_ld();
        if (tid < m) {
          float4 *dst = reinterpret_cast<float4 *>(a.vpart + ((long long)ks * a.T + row0 + tid) * a.r_cap);
#pragma unroll
          for (int q = 0; q < kPfRankCap / 4; ++q)
            if (q < R / 4) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
    }
    // the epilogue warps stay in step (an absent adapter's unit has no
    // other barrier that would hold them together)
    if (warp < kShEpiWarps) asm volatile("bar.sync 1, %0;" ::"n"(kShEpiThreads) : "memory");
    if (tid == 0) pf_arrive(S.stg_free);  // the staged slice may be overwritten
    gbase += nkb;
    if (use) ++ucount;
    ++ucopy;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kShTmemCols) : "memory");
  }
}

// ============================================================ expand kernel
struct ExSmem {
  uint8_t *ys, *bw, *vop;
  uint64_t *y_full, *mma_done;
  uint32_t *tmem_slot;
};

__host__ __device__ inline int ex_smem_bytes(int r_cap) {
  return 1024 /* alignment slack */ + kGroupBoxes * kBoxBytes + r_cap * kGroupCols * 2 + 2 * kMmaRows * r_cap * 2 +
         2 * 8 + 16;
}

// Every warp takes every step of a unit; several CTAs per SM overlap one's
// loads with another's epilogue.  Epilogue: warp w owns tile rows 32w .. +31
// and both y boxes of the unit.
__global__ void __launch_bounds__(kExThreads, kExMaxPerSm) pf_expand_kernel(const __grid_constant__ PrefillArgs a) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ExSmem S;
  {
    uint8_t *p = base;
    S.ys = p; p += kGroupBoxes * kBoxBytes;
    S.bw = p; p += a.r_cap * kGroupCols * 2;
    S.vop = p; p += 2 * kMmaRows * a.r_cap * 2;
    uint64_t *b = reinterpret_cast<uint64_t *>(p);
    S.y_full = b++;
    S.mma_done = b++;
    S.tmem_slot = reinterpret_cast<uint32_t *>(b);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(S.tmem_slot)),
                 "r"(kExTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    mbar_init(S.y_full, 1);
    mbar_init(S.mma_done, 1);
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_y)) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *S.tmem_slot;
  // The plan was complete before the shrink kernel let this one start, so
  // tiles, y and B^T may be read now; the partial V only after griddep_wait.
  bool waited = false;

  bool alive = true;
  const int n_units = a.hdr[kHdrTiles] * a.n_groups;
  const uint32_t lbo_b = (uint32_t)(kGroupCols / 8) * 128u;  // k-group stride of the B^T slice
  const uint32_t lbo_v = (uint32_t)(kMmaRows / 8) * 128u;    // k-group stride of V
  const uint32_t bw_u = smem_u32(S.bw), v_u = smem_u32(S.vop);
  uint32_t ucount = 0;

  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    const int tile = u / a.n_groups, grp = u - tile * a.n_groups;
    const int4 d = a.tiles[tile];
    // (LORA_DEBUG: a tile outside the pool's slots or the batch's rows is skipped by every role)
    if (!dbg_ok(d.x >= 0 && d.x < a.pool.n_slots && d.y >= 0 && d.z > 0 && d.z <= kMmaRows && d.y + d.z <= a.T,
                a.status))
      continue;
    const int slot = d.x, row0 = d.y, m = d.z;
    const int r = a.pool.rank[slot * a.pool.n_targets + a.target];
    const float scale = a.scales[slot];  // (read here: its latency overlaps the unit's loads)
    if (r <= 0 || r > a.r_cap) continue;  // reported by the shrink kernel
    const int R = (r + 15) & ~15;
    const uint32_t par = ucount & 1u;
    const int col_base = grp * kGroupCols;
    const int cols = min(kGroupCols, a.d_out - col_base);
    const int nbox = (cols + kBoxCols - 1) / kBoxCols;

    // (1) y boxes of the unit, by TMA
    if (tid == 0) {
      mbar_arrive_expect_tx(S.y_full, (uint32_t)(nbox * kBoxBytes));
      for (int b = 0; b < nbox; ++b)
        tma_load_2d(S.ys + b * kBoxBytes, &a.tmap_y, col_base + b * kBoxCols, row0, S.y_full);
    }
    // (2) B^T columns of the unit (rows < r; zero rows up to R and columns
    // beyond d_out) in the MMA's MN-major core-matrix layout
    // (chunks located through the pool's tiled arrangement of the block)
    const int bpage = block_page(a.pool, slot, a.bt_off, (long long)a.pool_r_max * a.d_out * 2);
    for (int idx = tid; idx < R * (kGroupCols / 8); idx += kExThreads) {
      const int jl = idx & 7, nv = (idx >> 3) & (kGroupCols / 8 - 1), jg = idx / (8 * (kGroupCols / 8));
      const int j = jg * 8 + jl;
      const uint32_t dst = bw_u + jg * lbo_b + nv * 128 + jl * 16;
      if (j < r && nv * 8 < cols)
        cp_async16_pf(dst, block_chunk(a.pool, slot, bpage,
                                       a.bt_off + block_chunk_off(j, col_base / 8 + nv, a.d_out, a.pool_r_max),
                                       a.status));
      else
        st_shared_zero16(dst);
    }
    // (3) V of the tile's row tid: the k-slice partials summed in fixed
    // order, as two bf16 operand terms
    if (!waited) {
      griddep_wait();
      griddep_launch_dependents();
      waited = true;
    }
    {
      const int i = tid;
      float v[kPfRankCap];
#pragma unroll
      for (int k = 0; k < kPfRankCap; ++k) v[k] = 0.f;
      if (i < m) {
        for (int s = 0; s < a.n_ks; ++s) {
          const float4 *src = reinterpret_cast<const float4 *>(a.vpart + ((long long)s * a.T + row0 + i) * a.r_cap);
#pragma unroll
          for (int q = 0; q < kPfRankCap / 4; ++q) {
            if (q < R / 4) {
              const float4 f = src[q];
              v[4 * q] += f.x;
              v[4 * q + 1] += f.y;
              v[4 * q + 2] += f.z;
              v[4 * q + 3] += f.w;
            }
          }
        }
      }
#pragma unroll
      for (int j8 = 0; j8 < kPfRankCap / 8; ++j8) {
        if (j8 >= R / 8) break;
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v0 = v[j8 * 8 + 2 * e], v1 = v[j8 * 8 + 2 * e + 1];
          hi[e] = pack_bf16x2(v0, v1);
          lo[e] = pack_bf16x2(v0 - bf16_lo(hi[e]), v1 - bf16_hi(hi[e]));
        }
        const uint32_t off = j8 * lbo_v + (i >> 3) * 128 + (i & 7) * 16;
        *reinterpret_cast<uint4 *>(S.vop + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(S.vop + (uint32_t)(R / 8) * lbo_v + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    cp_async_wait_all();
    fence_async_smem();  // generic-proxy writes -> visible to the MMAs (async proxy)
    __syncthreads();
    tc_fence_after();
    // (4) V (hi, lo) x B^T into TMEM (M 128, N 128, K = 2 R)
    if (tid == 0) {
      const uint32_t idesc_e = idesc_bf16(kChunkCols, true);
      bool first = true;
      for (int part = 0; part < 2; ++part) {
        for (int k16 = 0; k16 < R / 16; ++k16) {
          const uint64_t ad = smem_desc(v_u + (uint32_t)(part * (R / 8) + 2 * k16) * lbo_v, lbo_v, 128, 0);
          const uint64_t bd = smem_desc(bw_u + (uint32_t)(2 * k16) * lbo_b, lbo_b, 128, 0);
          mma_bf16(tmem, ad, bd, idesc_e, !first);
          first = false;
        }
      }
      mma_commit(S.mma_done);
    }
    // (5) epilogue
    warp_wait(S.mma_done, par, a.status, alive);
    warp_wait(S.y_full, par, a.status, alive);
    tc_fence_after();
    const int lg = warp;
    for (int b = 0; b < kGroupBoxes; ++b) {
      if (b >= nbox || !alive) break;  // warp-uniform
      float acc[64];
      const uint32_t taddr = tmem + ((uint32_t)(lg * 32) << 16) + (uint32_t)(b * kBoxCols);
      tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(acc));
      tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(acc + 16));
      tmem_ld16(taddr + 32, *reinterpret_cast<float(*)[16]>(acc + 32));
      tmem_ld16(taddr + 48, *reinterpret_cast<float(*)[16]>(acc + 48));
      tmem_wait_ld();
      uint8_t *box = S.ys + b * kBoxBytes;
      const int row = lg * 32 + lane;
      uint4 yv[8];
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) yv[c16] = *reinterpret_cast<const uint4 *>(box + row * 128 + ((c16 ^ (row & 7)) * 16));
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        float f[8];
        unpack8(yv[c16], f);
        uint4 o;
        o.x = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 0], f[0]), fmaf(scale, acc[c16 * 8 + 1], f[1]));
        o.y = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 2], f[2]), fmaf(scale, acc[c16 * 8 + 3], f[3]));
        o.z = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 4], f[4]), fmaf(scale, acc[c16 * 8 + 5], f[5]));
        o.w = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 6], f[6]), fmaf(scale, acc[c16 * 8 + 7], f[7]));
        *reinterpret_cast<uint4 *>(box + row * 128 + ((c16 ^ (row & 7)) * 16)) = o;
      }
      __syncwarp();
      // the warp's 32 rows out, 8 lanes per 128-byte row; only the tile's
      // own rows and columns inside d_out
      const int col0 = col_base + b * kBoxCols;
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int rl = lg * 32 + it * 4 + (lane >> 3), c = lane & 7;
        const int col = col0 + c * 8;
        if (rl < m && col < a.d_out) {
          const uint4 v = *reinterpret_cast<const uint4 *>(box + rl * 128 + ((c ^ (rl & 7)) * 16));
          *reinterpret_cast<uint4 *>(a.y + (long long)(row0 + rl) * a.ldy + col) = v;
        }
      }
    }
    fence_async_smem();  // the in-place y writes are ordered before the next unit's TMA writes
    tc_fence_before();
    __syncthreads();     // y boxes, B^T, V and TMEM are free for the next unit
    ++ucount;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kExTmemCols) : "memory");
  }
  if (!waited) {  // a CTA without units still orders the grids after it
    griddep_wait();
    griddep_launch_dependents();
  }
}

// ------------------------------------------------------------ host side
static bool make_map(CUtensorMap *map, const void *ptr, int cols, int rows, long long ld) {
  return make_tmap_2d(map, ptr, cols, rows, ld, kBoxCols, kMmaRows);
}

// Geometry of the two kernels for a target: the k-slice width (x blocks of
// 64 columns per shrink unit), the ring depth, the shared memory of each;
// false if the tensor-core path cannot serve this target (the decode kernel
// then takes the long segments too).  max_tiles bounds the tile count: few
// tiles get thinner k-slices so that the shrink still spreads over the SMs.
bool prefill_geometry(const lora_pool *pool, int target, int max_tiles, PrefillGeometry *g) {
  if (pool->r_max > kPfRankCap) return false;
  const int d_in = pool->targets[target].d_in, d_out = pool->targets[target].d_out;
  const int r_cap = pool->r_max <= 16 ? 16 : 32;
  const int nkb_all = (d_in + kBoxCols - 1) / kBoxCols;
  const int want_ks = std::max(1, (kSms + std::max(max_tiles, 1) - 1) / std::max(max_tiles, 1));
  // k-slices of whole pool tiles (the shrink copies its adapter slice one
  // tile at a time)
  const int tb = pool_tile_cols(pool->r_max) / kBoxCols;
  int kb_per = (nkb_all + want_ks - 1) / want_ks;
  kb_per = std::max(tb, std::min(kShMaxBlocks, (kb_per + tb - 1) / tb * tb));
  kb_per = std::min(kb_per, nkb_all);
  const int cap = 227 * 1024;
  int ns = 0;
  for (int st = kShMaxStages; st >= 2; --st)
    if (sh_smem_bytes(st, r_cap, kb_per) <= cap) {
      ns = st;
      break;
    }
  if (ns == 0) return false;
  g->r_cap = r_cap;
  g->kb_per = kb_per;
  g->n_ks = (nkb_all + kb_per - 1) / kb_per;
  g->n_stages = ns;
  g->smem_sh = sh_smem_bytes(ns, r_cap, kb_per);
  g->smem_ex = ex_smem_bytes(r_cap);
  g->n_groups = (d_out + kGroupCols - 1) / kGroupCols;
  return g->smem_ex <= cap;
}

size_t prefill_scratch_bytes(const lora_pool *pool, int target, int T) {
  PrefillGeometry g;
  if (T <= 0 || !prefill_geometry(pool, target, plan_layout(T).j_max, &g)) return 0;
  return align256(size_t(T) * g.n_ks * g.r_cap * 4);
}

static int pool_sms(const lora_pool *pool) {
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, pool->device) != cudaSuccess) {
    (void)cudaGetLastError();
    return kSms;
  }
  return sms;
}

template <typename K>
static int co_resident(lora_pool *pool, K kernel, int key, int threads, int smem) {
  std::lock_guard<std::mutex> lk(pool->mu);
  auto k = std::make_pair(key, smem);
  auto it = pool->prefill_fit.find(k);
  if (it != pool->prefill_fit.end()) return it->second;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, pool->device) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  pool->prefill_fit[k] = per_sm * sms;
  return per_sm * sms;
}

int launch_prefill(lora_pool *pool, int target, const void *x, int ldx, void *y, int ldy, const float *scales,
                   int T, const void *ws, size_t ws_bytes, cudaStream_t st) {
  PlanLayout L = plan_layout(T);
  PrefillGeometry geo;
  if (!prefill_geometry(pool, target, L.j_max, &geo)) return LORA_ERR_INVALID_ARG;
  const size_t plan_bytes = align256(L.total);
  if (ws_bytes < plan_bytes + prefill_scratch_bytes(pool, target, T)) return LORA_ERR_WORKSPACE;
  PlanView pv = plan_view(const_cast<void *>(ws), L);
  PrefillArgs a;
  memset(&a, 0, sizeof(a));
  const int d_in = pool->targets[target].d_in, d_out = pool->targets[target].d_out;
  if (!make_map(&a.tmap_x, x, d_in, T, ldx) || !make_map(&a.tmap_y, y, d_out, T, ldy)) return LORA_ERR_CUDA;
  a.pool = pool->view();
  a.target = target;
  a.d_in = d_in;
  a.d_out = d_out;
  a.T = T;
  a.a_off = pool->a_off[target];
  a.bt_off = pool->bt_off[target];
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.scales = scales;
  a.hdr = pv.hdr;
  a.tiles = pv.tiles;
  a.status = pool->d_status;
  a.vpart = reinterpret_cast<float *>(static_cast<uint8_t *>(const_cast<void *>(ws)) + plan_bytes);
  a.r_cap = geo.r_cap;
  a.pool_r_max = pool->r_max;
  a.kb_per = geo.kb_per;
  a.n_ks = geo.n_ks;
  a.n_stages = geo.n_stages;
  a.n_groups = geo.n_groups;

  static int attr_done[64] = {};
  if (pool->device < 0 || pool->device >= 64) return LORA_ERR_INVALID_ARG;
  if (!attr_done[pool->device]) {
    // the largest shared-memory carveout, so that several expand CTAs fit per SM
    if (cudaFuncSetAttribute(pf_shrink_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(pf_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ex_smem_bytes(kPfRankCap)) != cudaSuccess ||
        cudaFuncSetAttribute(pf_shrink_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
        cudaFuncSetAttribute(pf_expand_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return LORA_ERR_CUDA;
    attr_done[pool->device] = 1;
  }
  const int fit_sh = co_resident(pool, pf_shrink_kernel, 1, kShThreads, geo.smem_sh);
  if (fit_sh < 1) return LORA_ERR_CUDA;
  // expand CTAs per SM: bounded by shared memory and by TMEM (kExMaxPerSm)
  const int fit_ex = std::max(1, std::min(kExMaxPerSm, kSmemPerSm / (geo.smem_ex + 1024))) * pool_sms(pool);
  // one wave of CTAs that loop over the units (tiles <= L.j_max)
  const long long units_sh = (long long)L.j_max * geo.n_ks, units_ex = (long long)L.j_max * geo.n_groups;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cudaLaunchConfig_t cfg = {};
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)std::min<long long>(units_sh, fit_sh));
  cfg.blockDim = dim3(kShThreads);
  cfg.dynamicSmemBytes = geo.smem_sh;
  g_launches.fetch_add(1);
  if (cudaLaunchKernelEx(&cfg, pf_shrink_kernel, a) != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  cfg.gridDim = dim3((unsigned)std::min<long long>(units_ex, fit_ex));
  cfg.blockDim = dim3(kExThreads);
  cfg.dynamicSmemBytes = geo.smem_ex;
  g_launches.fetch_add(1);
  if (cudaLaunchKernelEx(&cfg, pf_expand_kernel, a) != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

}  // namespace lora
