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
// B200 mapping.  A cluster of C CTAs (4 or 8) owns one 128-row tile.  CTA c
// streams its slice of d_in of the tile's x rows with TMA (2-D tiled loads,
// 128-byte swizzle, no multicast) and accumulates its split-K share of V in
// TMEM with tcgen05.mma (kind::f16, bf16 in, fp32 accumulate); the adapter
// rows sit in shared memory, copied once per tile through the page table.
// Shares of V are summed over the cluster through distributed shared memory
// in fixed CTA order, V is split into two bf16 terms (hi + lo, about 16 bits
// of V kept) and CTA c expands its slice of d_out in 128-column chunks into
// two TMEM buffers, so the MMA of one chunk overlaps the epilogue of the
// other.  The epilogue adds s * acc to y (prefetched by TMA) in fp32 and
// stores bf16 for the tile's own rows only.  One thread issues TMA and MMA;
// all waits are bounded.
#include <cooperative_groups.h>
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "internal.cuh"

namespace cg = cooperative_groups;

namespace lora {

constexpr int kPfThreads = 128;
constexpr int kPfMaxStages = 4;
constexpr int kBoxCols = 64;                 // TMA box: 64 bf16 (128 B) x 128 rows
constexpr int kBoxBytes = kBoxCols * 2 * kMmaRows;
constexpr int kChunkCols = 128;              // expand MMA N
constexpr int kTmemCols = 256;               // two expand buffers; shrink uses [0, R)
constexpr int kPfRankCap = 32;

struct __align__(64) PrefillArgs {
  CUtensorMap tmap_x;   // x [T, d_in], box 64 x 128, 128-byte swizzle
  CUtensorMap tmap_y;   // y [T, d_out], same box
  PoolView pool;
  int target, d_in, d_out;
  long long a_off, bt_off;
  uint16_t *y;
  long long ldy;
  const float *scales;
  const int32_t *hdr;
  const int4 *tiles;
  int *status;
  int ks_cols;          // shared-memory columns of the A_a slice (multiple of 64)
  int ns_cols;          // shared-memory columns of the B^T slice (multiple of 128)
  int r_cap;            // 16 or 32: rank rows held per slice
  int nsx, nsy;         // x and y pipeline depths
};

// ------------------------------------------------------------ tcgen05 / TMA
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// kind::f16 instruction descriptor: bf16 A and B, fp32 D, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(kMmaRows >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)acc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Bounded wait that gives up for good once one wait of this thread failed.
__device__ __forceinline__ bool pf_wait(uint64_t *bar, uint32_t parity, int *status, bool &alive) {
  if (!alive) return false;
  if (!mbar_wait_bounded(bar, parity, status)) alive = false;
  return alive;
}

struct PfSmem {
  uint8_t *xs, *ys, *aw, *bw, *vop;
  float *part;
  uint64_t *x_full, *x_empty, *y_full, *sh_done, *ex_done;
  uint32_t *tmem_slot;
};

__device__ __forceinline__ PfSmem pf_carve(uint8_t *base, const PrefillArgs &a) {
  PfSmem s;
  uint8_t *p = base;
  s.xs = p; p += a.nsx * kBoxBytes;
  s.ys = p; p += a.nsy * kBoxBytes;
  s.aw = p; p += a.r_cap * a.ks_cols * 2;
  s.bw = p; p += a.r_cap * a.ns_cols * 2;
  s.vop = p; p += 2 * kMmaRows * a.r_cap * 2;
  s.part = reinterpret_cast<float *>(p); p += kMmaRows * a.r_cap * 4;
  uint64_t *b = reinterpret_cast<uint64_t *>(p);
  s.x_full = b; b += kPfMaxStages;
  s.x_empty = b; b += kPfMaxStages;
  s.y_full = b; b += kPfMaxStages;
  s.sh_done = b; b += 1;
  s.ex_done = b; b += 2;
  s.tmem_slot = reinterpret_cast<uint32_t *>(b);
  return s;
}

__host__ __device__ inline int pf_smem_bytes(int nsx, int nsy, int r_cap, int ks_cols, int ns_cols) {
  return 1024 /* alignment slack */ + (nsx + nsy) * kBoxBytes + r_cap * (ks_cols + ns_cols) * 2 +
         2 * kMmaRows * r_cap * 2 + kMmaRows * r_cap * 4 + (3 * kPfMaxStages + 3) * 8 + 16;
}

__global__ void __launch_bounds__(kPfThreads, 1) prefill_kernel(const __grid_constant__ PrefillArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int cid = blockIdx.x / C, ncl = gridDim.x / C;
  const int tid = threadIdx.x, warp = tid >> 5;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PfSmem S = pf_carve(base, a);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(S.tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < kPfMaxStages; ++i) {
      mbar_init(&S.x_full[i], 1);
      mbar_init(&S.x_empty[i], 1);
      mbar_init(&S.y_full[i], 1);
    }
    mbar_init(S.sh_done, 1);
    mbar_init(&S.ex_done[0], 1);
    mbar_init(&S.ex_done[1], 1);
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_y)) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *S.tmem_slot;
  griddep_wait();

  bool alive = true;
  const int n_tiles = a.hdr[kHdrTiles];
  const int nkb_all = (a.d_in + kBoxCols - 1) / kBoxCols;
  const int nq_all = (a.d_out + kChunkCols - 1) / kChunkCols;
  const int kb_per = (nkb_all + C - 1) / C, q_per = (nq_all + C - 1) / C;
  const int kb0 = min(crank * kb_per, nkb_all), kb1 = min(kb0 + kb_per, nkb_all);
  const int q0 = min(crank * q_per, nq_all), q1 = min(q0 + q_per, nq_all);
  const int nkb = kb1 - kb0, nq = q1 - q0;
  const uint32_t lbo_a = (uint32_t)(a.r_cap / 8) * 128u;          // k-group stride of the A_a slice
  const uint32_t lbo_b = (uint32_t)(a.ns_cols / 8) * 128u;        // k-group stride of the B^T slice
  const uint32_t lbo_v = (uint32_t)(kMmaRows / 8) * 128u;         // k-group stride of V
  const uint32_t aw_u = smem_u32(S.aw), bw_u = smem_u32(S.bw), v_u = smem_u32(S.vop);

  // Phase / stage counters: x stages are consumed by thread 0 only; the
  // y stages, sh_done and ex_done by every thread, identically.
  uint32_t gx = 0, gy = 0, sh_phase = 0, ex_phase[2] = {0, 0};

  for (int tile = cid; tile < n_tiles; tile += ncl) {
    const int4 d = a.tiles[tile];
    const int slot = d.x, row0 = d.y, m = d.z;
    const int r = a.pool.rank[slot * a.pool.n_targets + a.target];
    if (r <= 0 || r > a.r_cap) {
      if (r > a.r_cap && tid == 0) set_status(a.status, LORA_ERR_INVALID_ARG);
      continue;
    }
    const int R = (r + 15) & ~15;
    const float scale = a.scales[slot];
    const int n_ybox = 2 * nq;
    const uint32_t ybase = gy;  // y box i of this tile uses stage (ybase + i) % nsy

    // ---- producer prologue: the first x blocks and y boxes of this tile
    if (tid == 0) {
      for (int i = 0; i < nkb && i < a.nsx; ++i) {
        const uint32_t g = gx + i, st = g % a.nsx;
        if (g >= (uint32_t)a.nsx) pf_wait(&S.x_empty[st], ((g / a.nsx) - 1) & 1, a.status, alive);
        mbar_arrive_expect_tx(&S.x_full[st], kBoxBytes);
        tma_load_2d(S.xs + st * kBoxBytes, &a.tmap_x, (kb0 + i) * kBoxCols, row0, &S.x_full[st]);
      }
      for (int i = 0; i < n_ybox && i < a.nsy; ++i) {
        const uint32_t st = (ybase + i) % a.nsy;
        const int q = q0 + i / 2, h = i % 2;
        mbar_arrive_expect_tx(&S.y_full[st], kBoxBytes);
        tma_load_2d(S.ys + st * kBoxBytes, &a.tmap_y, q * kChunkCols + h * kBoxCols, row0, &S.y_full[st]);
      }
    }

    // ---- adapter rows of this tile into shared memory (zero beyond rank / edge)
    {
      const int kv_n = a.ks_cols / 8;
      for (int idx = tid; idx < a.r_cap * kv_n; idx += kPfThreads) {
        const int j = idx / kv_n, kv = idx - j * kv_n, k = kb0 * kBoxCols + kv * 8;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (j < r && k < a.d_in && kv < nkb * (kBoxCols / 8)) {
          long long room;
          const uint8_t *src = pool_addr(a.pool, slot, a.a_off + ((long long)j * a.d_in + k) * 2, &room);
          if (src) val = *reinterpret_cast<const uint4 *>(src);
        }
        *reinterpret_cast<uint4 *>(S.aw + kv * lbo_a + (j >> 3) * 128 + (j & 7) * 16) = val;
      }
      const int nv_n = a.ns_cols / 8;
      for (int idx = tid; idx < a.r_cap * nv_n; idx += kPfThreads) {
        const int j = idx / nv_n, nv = idx - j * nv_n, n = q0 * kChunkCols + nv * 8;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (j < r && n < a.d_out && nv < nq * (kChunkCols / 8)) {
          long long room;
          const uint8_t *src = pool_addr(a.pool, slot, a.bt_off + ((long long)j * a.d_out + n) * 2, &room);
          if (src) val = *reinterpret_cast<const uint4 *>(src);
        }
        *reinterpret_cast<uint4 *>(S.bw + (j >> 3) * lbo_b + nv * 128 + (j & 7) * 16) = val;
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- shrink: V_part[128 x R] = X[:, slice] A_a[:R, slice]^T in TMEM columns [0, R)
    if (tid == 0) {
      const uint32_t idesc = idesc_bf16(R, false);
      for (int i = 0; i < nkb; ++i) {
        const uint32_t g = gx + i, st = g % a.nsx;
        pf_wait(&S.x_full[st], (g / a.nsx) & 1, a.status, alive);
        tc_fence_after();
        const uint32_t xa = smem_u32(S.xs + st * kBoxBytes);
#pragma unroll
        for (int kk = 0; kk < kBoxCols / 16; ++kk) {
          const uint64_t ad = smem_desc(xa + kk * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(aw_u + (uint32_t)(i * 4 + kk) * 2 * lbo_a, lbo_a, 128, 0);
          if (alive) mma_bf16(tmem, ad, bd, idesc, (i | kk) != 0);
        }
        mma_commit(&S.x_empty[st]);
        if (i + a.nsx < nkb) {  // refill this stage with block i + nsx once its MMAs are done
          pf_wait(&S.x_empty[st], (g / a.nsx) & 1, a.status, alive);
          mbar_arrive_expect_tx(&S.x_full[st], kBoxBytes);
          tma_load_2d(S.xs + st * kBoxBytes, &a.tmap_x, (kb0 + i + a.nsx) * kBoxCols, row0, &S.x_full[st]);
        }
      }
      mma_commit(S.sh_done);
    }
    // the stages whose refill was not waited for are released by their
    // commits; account for them so the next tile's prologue waits correctly
    gx += nkb;

    // ---- this CTA's share of V -> registers -> shared memory
    pf_wait(S.sh_done, sh_phase, a.status, alive);
    sh_phase ^= 1;
    tc_fence_after();
    float vrow[kPfRankCap];
#pragma unroll
    for (int j = 0; j < kPfRankCap; ++j) vrow[j] = 0.f;
    if (nkb > 0) {
      const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
      float t16[16];
      tmem_ld16(lane_addr + 0, t16);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) vrow[j] = t16[j];
      if (R > 16) {
        tmem_ld16(lane_addr + 16, t16);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) vrow[16 + j] = t16[j];
      }
    }
    for (int j = 0; j < R; ++j) S.part[tid * a.r_cap + j] = vrow[j];
    tc_fence_before();

    // ---- sum the shares over the cluster (fixed CTA order), split into bf16 hi + lo
    cluster.sync();
    for (int j = 0; j < R; ++j) vrow[j] = 0.f;
    for (int c = 0; c < C; ++c) {
      const float *rp = cluster.map_shared_rank(S.part, c) + tid * a.r_cap;
      for (int j = 0; j < R; ++j) vrow[j] += rp[j];
    }
    cluster.sync();
    for (int j8 = 0; j8 < R / 8; ++j8) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v0 = vrow[j8 * 8 + 2 * e], v1 = vrow[j8 * 8 + 2 * e + 1];
        hi[e] = pack_bf16x2(v0, v1);
        lo[e] = pack_bf16x2(v0 - bf16_lo(hi[e]), v1 - bf16_hi(hi[e]));
      }
      const uint32_t off = j8 * lbo_v + (tid >> 3) * 128 + (tid & 7) * 16;
      *reinterpret_cast<uint4 *>(S.vop + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4 *>(S.vop + (uint32_t)(R / 8) * lbo_v + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- expand: 128-column chunks into alternating TMEM buffers
    const uint32_t idesc_e = idesc_bf16(kChunkCols, true);
    auto issue_expand = [&](int q) {
      const uint32_t buf = tmem + (uint32_t)((q & 1) * kChunkCols);
      const uint32_t b_chunk = bw_u + (uint32_t)q * (kChunkCols / 8) * 128;
      bool first = true;
      for (int part = 0; part < 2; ++part) {
        for (int ks = 0; ks < R / 16; ++ks) {
          const uint64_t ad = smem_desc(v_u + (uint32_t)(part * (R / 8) + 2 * ks) * lbo_v, lbo_v, 128, 0);
          const uint64_t bd = smem_desc(b_chunk + (uint32_t)(2 * ks) * lbo_b, lbo_b, 128, 0);
          if (alive) mma_bf16(buf, ad, bd, idesc_e, !first);
          first = false;
        }
      }
      mma_commit(&S.ex_done[q & 1]);
    };
    if (tid == 0 && nq > 0) issue_expand(0);
    for (int q = 0; q < nq; ++q) {
      if (tid == 0 && q + 1 < nq) issue_expand(q + 1);
      pf_wait(&S.ex_done[q & 1], ex_phase[q & 1], a.status, alive);
      ex_phase[q & 1] ^= 1;
      tc_fence_after();
      for (int h = 0; h < 2; ++h) {
        const uint32_t st = gy % a.nsy;
        pf_wait(&S.y_full[st], (gy / a.nsy) & 1, a.status, alive);
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)((q & 1) * kChunkCols + h * kBoxCols);
        float acc[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float t16[16];
          tmem_ld16(lane_addr + c * 16, t16);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[c * 16 + e] = t16[e];
        }
        const int col0 = (q0 + q) * kChunkCols + h * kBoxCols;
        if (tid < m) {
          const uint8_t *yrow = S.ys + st * kBoxBytes + tid * 128;
          uint16_t *dst = a.y + (long long)(row0 + tid) * a.ldy + col0;
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {
            if (col0 + c16 * 8 >= a.d_out) break;
            const uint4 u = *reinterpret_cast<const uint4 *>(yrow + ((c16 ^ (tid & 7)) * 16));
            float yv[8];
            unpack8(u, yv);
            uint4 o;
            o.x = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 0], yv[0]), fmaf(scale, acc[c16 * 8 + 1], yv[1]));
            o.y = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 2], yv[2]), fmaf(scale, acc[c16 * 8 + 3], yv[3]));
            o.z = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 4], yv[4]), fmaf(scale, acc[c16 * 8 + 5], yv[5]));
            o.w = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 6], yv[6]), fmaf(scale, acc[c16 * 8 + 7], yv[7]));
            *reinterpret_cast<uint4 *>(dst + c16 * 8) = o;
          }
        }
        __syncthreads();  // y stage consumed
        if (tid == 0 && q * 2 + h + a.nsy < n_ybox) {  // refill it with box j + nsy of this tile
          const int i2 = q * 2 + h + a.nsy;
          mbar_arrive_expect_tx(&S.y_full[st], kBoxBytes);
          tma_load_2d(S.ys + st * kBoxBytes, &a.tmap_y, (q0 + i2 / 2) * kChunkCols + (i2 % 2) * kBoxCols, row0,
                      &S.y_full[st]);
        }
        ++gy;
      }
      tc_fence_before();
      __syncthreads();  // TMEM buffer q & 1 is free again
      tc_fence_after();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  griddep_launch_dependents();
}

// ------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    (void)cudaGetLastError();
  });
  return fn;
}

static bool make_map(CUtensorMap *map, const void *ptr, int cols, int rows, long long ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {kBoxCols, kMmaRows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pick the cluster size and pipeline depths that fit shared memory; false if
// the tensor-core path cannot serve this target (the decode kernel then takes
// the long segments too).
bool prefill_geometry(const lora_pool *pool, int target, PrefillGeometry *g) {
  if (pool->r_max > kPfRankCap) return false;
  const int d_in = pool->targets[target].d_in, d_out = pool->targets[target].d_out;
  const int r_cap = pool->r_max <= 16 ? 16 : 32;
  const int nkb_all = (d_in + kBoxCols - 1) / kBoxCols, nq_all = (d_out + kChunkCols - 1) / kChunkCols;
  const int cap = 227 * 1024;
  for (int C : {4, 8}) {
    const int ks = ((nkb_all + C - 1) / C) * kBoxCols, ns = ((nq_all + C - 1) / C) * kChunkCols;
    for (int st = 4; st >= 2; --st) {
      const int smem = pf_smem_bytes(st, st, r_cap, ks, ns);
      if (smem <= cap) {
        *g = {C, st, st, r_cap, ks, ns, smem};
        return true;
      }
    }
  }
  return false;
}

int launch_prefill(lora_pool *pool, int target, const void *x, int ldx, void *y, int ldy, const float *scales,
                   int T, const void *ws, cudaStream_t st) {
  PrefillGeometry geo;
  if (!prefill_geometry(pool, target, &geo)) return LORA_ERR_INVALID_ARG;
  PlanLayout L = plan_layout(T);
  PlanView pv = plan_view(const_cast<void *>(ws), L);
  PrefillArgs a;
  memset(&a, 0, sizeof(a));
  const int d_in = pool->targets[target].d_in, d_out = pool->targets[target].d_out;
  if (!make_map(&a.tmap_x, x, d_in, T, ldx) || !make_map(&a.tmap_y, y, d_out, T, ldy)) return LORA_ERR_CUDA;
  a.pool = pool->view();
  a.target = target;
  a.d_in = d_in;
  a.d_out = d_out;
  a.a_off = pool->a_off[target];
  a.bt_off = pool->bt_off[target];
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.scales = scales;
  a.hdr = pv.hdr;
  a.tiles = pv.tiles;
  a.status = pool->d_status;
  a.ks_cols = geo.ks_cols;
  a.ns_cols = geo.ns_cols;
  a.r_cap = geo.r_cap;
  a.nsx = geo.nsx;
  a.nsy = geo.nsy;

  static int attr_smem[64] = {};
  if (pool->device < 64 && attr_smem[pool->device] < geo.smem) {
    if (cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
        cudaSuccess)
      return LORA_ERR_CUDA;
    attr_smem[pool->device] = 227 * 1024;
  }
  // tiles <= T / 128 + number of long segments; clusters loop over tiles
  const int max_tiles = L.j_max;
  const int sms = 148;
  int n_clusters = std::max(1, std::min(max_tiles, sms / geo.C));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_clusters * geo.C);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = geo.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = geo.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  g_launches.fetch_add(1);
  if (cudaLaunchKernelEx(&cfg, prefill_kernel, a) != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

}  // namespace lora
