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

constexpr int kPfEpiWarps = 4;
constexpr int kPfEpiThreads = 32 * kPfEpiWarps;
constexpr int kPfThreads = kPfEpiThreads + 64;  // + TMA producer warp + MMA warp
constexpr int kPfMaxStages = 12;
constexpr int kBoxCols = 64;                 // TMA box: 64 bf16 (128 B) x 128 rows
constexpr int kBoxBytes = kBoxCols * 2 * kMmaRows;
constexpr int kChunkCols = 128;              // expand MMA N
constexpr int kTmemCols = 512;               // two expand buffers [0, 256); the shrink share at kVCol
constexpr uint32_t kVCol = 256;
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
  int n_stages;         // stages of the x / y box ring
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

// Remote mbarrier arrive on the same barrier of CTA `cta` of the cluster
// (release at cluster scope: this warp's prior shared-memory writes and reads
// are ordered before it).
__device__ __forceinline__ void mbar_arrive_remote(uint64_t *bar, uint32_t cta) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(bar)), "r"(cta));
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t *bar, uint32_t parity) {
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
__device__ __forceinline__ bool pf_wait_cluster(uint64_t *bar, uint32_t parity, int *status, bool &alive) {
  if (!alive) return false;
  if (mbar_try_wait_acq_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    if ((i & 255u) == 255u && global_timer_ns() - t0 > kSpinNs) break;
  }
  set_status(status, LORA_ERR_TIMEOUT);
  alive = false;
  return false;
}
// Epilogue waits: every lane waits (each acquires the data itself), then the
// warp agrees, so warp-collective tcgen05 loads stay convergent.
__device__ __forceinline__ bool epi_wait(uint64_t *bar, uint32_t parity, int *status, bool &alive) {
  pf_wait(bar, parity, status, alive);
  alive = __all_sync(0xffffffffu, alive);
  return alive;
}
__device__ __forceinline__ bool epi_wait_cluster(uint64_t *bar, uint32_t parity, int *status, bool &alive) {
  pf_wait_cluster(bar, parity, status, alive);
  alive = __all_sync(0xffffffffu, alive);
  return alive;
}
__device__ __forceinline__ void pf_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async16_pf(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Barrier of the four epilogue warps only (named barrier 1).
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kPfEpiThreads) : "memory"); }

struct PfSmem {
  uint8_t *ring, *aw, *bw, *vop;
  float *part;
  const uint8_t **arow, **brow;  // per rank row: start of this CTA's slice, or null (crosses a page)
  uint64_t *full, *empty;        // [kPfMaxStages]
  uint64_t *w_full, *sh_done, *v_full, *part_ready, *part_free;
  uint64_t *ex_done, *ex_free;   // [2]
  uint32_t *tmem_slot;
};

__device__ __forceinline__ PfSmem pf_carve(uint8_t *base, const PrefillArgs &a) {
  PfSmem s;
  uint8_t *p = base;
  s.ring = p; p += a.n_stages * kBoxBytes;
  s.aw = p; p += a.r_cap * a.ks_cols * 2;
  s.bw = p; p += a.r_cap * a.ns_cols * 2;
  s.vop = p; p += 2 * kMmaRows * a.r_cap * 2;
  s.part = reinterpret_cast<float *>(p); p += kMmaRows * a.r_cap * 4;
  s.arow = reinterpret_cast<const uint8_t **>(p); p += kPfRankCap * 8;
  s.brow = reinterpret_cast<const uint8_t **>(p); p += kPfRankCap * 8;
  uint64_t *b = reinterpret_cast<uint64_t *>(p);
  s.full = b; b += kPfMaxStages;
  s.empty = b; b += kPfMaxStages;
  s.w_full = b++;
  s.sh_done = b++;
  s.v_full = b++;
  s.part_ready = b++;
  s.part_free = b++;
  s.ex_done = b; b += 2;
  s.ex_free = b; b += 2;
  s.tmem_slot = reinterpret_cast<uint32_t *>(b);
  return s;
}

__host__ __device__ inline int pf_smem_bytes(int n_stages, int r_cap, int ks_cols, int ns_cols) {
  return 1024 /* alignment slack */ + n_stages * kBoxBytes + r_cap * (ks_cols + ns_cols) * 2 +
         2 * kMmaRows * r_cap * 2 + kMmaRows * r_cap * 4 + 2 * kPfRankCap * 8 + (2 * kPfMaxStages + 9) * 8 + 16;
}

// Warp roles: warps 0-3 copy the adapter slices, reduce V over the cluster
// and run the epilogue (warp w owns TMEM lanes / tile rows 32w .. 32w + 31);
// warp 4 issues the TMA loads of x blocks and y boxes into one stage ring;
// warp 5 issues the tensor-core MMAs.  Every role walks the same tile list.
__global__ void __launch_bounds__(kPfThreads, 1) prefill_kernel(const __grid_constant__ PrefillArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int cid = blockIdx.x / C, ncl = gridDim.x / C;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NS = a.n_stages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PfSmem S = pf_carve(base, a);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(S.tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == kPfEpiThreads) {
    for (int i = 0; i < kPfMaxStages; ++i) {
      mbar_init(&S.full[i], 1);
      mbar_init(&S.empty[i], 1);
    }
    mbar_init(S.w_full, kPfEpiThreads);
    mbar_init(S.sh_done, 1);
    mbar_init(S.v_full, kPfEpiThreads);
    mbar_init(S.part_ready, kPfEpiWarps * C);
    mbar_init(S.part_free, kPfEpiWarps * C);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.ex_done[i], 1);
      mbar_init(&S.ex_free[i], kPfEpiWarps);
    }
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_y)) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // every CTA's barriers are initialised before any peer arrives on them
  cluster.sync();
  const uint32_t tmem = *S.tmem_slot;
  griddep_wait();

  bool alive = true;
  const int n_tiles = a.hdr[kHdrTiles];
  const int nkb_all = (a.d_in + kBoxCols - 1) / kBoxCols;
  const int nq_all = (a.d_out + kChunkCols - 1) / kChunkCols;
  const int kb_per = (nkb_all + C - 1) / C, q_per = (nq_all + C - 1) / C;
  const int kb0 = min(crank * kb_per, nkb_all), kb1 = min(kb0 + kb_per, nkb_all);
  const int q0 = min(crank * q_per, nq_all), q1 = min(q0 + q_per, nq_all);
  const int nkb = kb1 - kb0, nq = q1 - q0, n_ybox = 2 * nq;
  const uint32_t lbo_a = (uint32_t)(a.r_cap / 8) * 128u;    // k-group stride of the A_a slice
  const uint32_t lbo_b = (uint32_t)(a.ns_cols / 8) * 128u;  // k-group stride of the B^T slice
  const uint32_t lbo_v = (uint32_t)(kMmaRows / 8) * 128u;   // k-group stride of V
  const uint32_t aw_u = smem_u32(S.aw), bw_u = smem_u32(S.bw), v_u = smem_u32(S.vop);
  const uint32_t ring_u = smem_u32(S.ring);

  // Ring sequence: each tile puts its nkb x blocks, then its n_ybox y boxes,
  // through the ring; use g sits in stage g % NS with phase (g / NS) & 1.
  uint32_t gbase = 0, ge = 0;  // ring uses and expand chunks so far (identical in every role)
  uint32_t tcount = 0;         // tiles done (per-tile barrier phases)

  for (int tile = cid; tile < n_tiles; tile += ncl) {
    const int4 d = a.tiles[tile];
    const int slot = d.x, row0 = d.y, m = d.z;
    const int r = a.pool.rank[slot * a.pool.n_targets + a.target];
    if (r <= 0 || r > a.r_cap) {
      if (r > a.r_cap && tid == 0) set_status(a.status, LORA_ERR_INVALID_ARG);
      continue;
    }
    const int R = (r + 15) & ~15;
    const uint32_t tpar = tcount & 1u;

    if (warp == kPfEpiWarps) {
      // ------------------------------------------------ TMA producer
      if (lane == 0) {
        for (int i = 0; i < nkb + n_ybox; ++i) {
          const uint32_t g = gbase + i, st = g % NS;
          if (g >= (uint32_t)NS && !pf_wait(&S.empty[st], ((g / NS) - 1) & 1, a.status, alive)) break;
          mbar_arrive_expect_tx(&S.full[st], kBoxBytes);
          if (i < nkb) {
            tma_load_2d(S.ring + st * kBoxBytes, &a.tmap_x, (kb0 + i) * kBoxCols, row0, &S.full[st]);
          } else {
            const int j = i - nkb;
            tma_load_2d(S.ring + st * kBoxBytes, &a.tmap_y, (q0 + j / 2) * kChunkCols + (j % 2) * kBoxCols, row0,
                        &S.full[st]);
          }
        }
      }
      __syncwarp();
    } else if (warp == kPfEpiWarps + 1) {
      // ------------------------------------------------ MMA issuer
      if (lane == 0) {
        pf_wait(S.w_full, tpar, a.status, alive);
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(R, false);
        for (int i = 0; i < nkb; ++i) {
          const uint32_t g = gbase + i, st = g % NS;
          pf_wait(&S.full[st], (g / NS) & 1, a.status, alive);
          tc_fence_after();
          const uint32_t xa = ring_u + st * kBoxBytes;
#pragma unroll
          for (int kk = 0; kk < kBoxCols / 16; ++kk) {
            const uint64_t ad = smem_desc(xa + kk * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(aw_u + (uint32_t)(i * 4 + kk) * 2 * lbo_a, lbo_a, 128, 0);
            if (alive) mma_bf16(tmem + kVCol, ad, bd, idesc, (i | kk) != 0);
          }
          mma_commit(&S.empty[st]);  // the stage is free once these MMAs have read it
        }
        mma_commit(S.sh_done);
        pf_wait(S.v_full, tpar, a.status, alive);
        tc_fence_after();
        const uint32_t idesc_e = idesc_bf16(kChunkCols, true);
        for (int q = 0; q < nq; ++q) {
          const uint32_t e = ge + q, b = e & 1u, u = e >> 1;
          if (u >= 1) pf_wait(&S.ex_free[b], (u - 1) & 1, a.status, alive);
          tc_fence_after();
          const uint32_t buf = tmem + b * kChunkCols;
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
          mma_commit(&S.ex_done[b]);
        }
      }
      __syncwarp();
    } else {
      // ------------------------------------------------ epilogue warps
      // (1) adapter slices of this tile -> shared memory, in the MMA's
      // no-swizzle core-matrix layouts; ranks r .. R-1 and columns beyond the
      // slice are zero.  Row starts are looked up once per row.
      const int ks_valid = min(nkb * kBoxCols, a.d_in - kb0 * kBoxCols);   // columns of this CTA's d_in slice
      const int ns_valid = min(nq * kChunkCols, a.d_out - q0 * kChunkCols);
      // (a row start is looked up only when the slice is not empty: the lookup
      // must stay inside the slot's pages)
      if (tid < r && ks_valid > 0) {
        long long room;
        const uint8_t *p = pool_addr(a.pool, slot, a.a_off + ((long long)tid * a.d_in + kb0 * kBoxCols) * 2, &room);
        S.arow[tid] = (p && room >= (long long)ks_valid * 2) ? p : nullptr;
      } else if (tid >= 64 && tid < 64 + r && ns_valid > 0) {
        const int j = tid - 64;
        long long room;
        const uint8_t *p = pool_addr(a.pool, slot, a.bt_off + ((long long)j * a.d_out + q0 * kChunkCols) * 2, &room);
        S.brow[j] = (p && room >= (long long)ns_valid * 2) ? p : nullptr;
      }
      epi_sync();
      const int jl = lane & 7, vo = lane >> 3;  // 8 rank rows x 4 consecutive 16-byte chunks per warp access
      const int kv_n = a.ks_cols / 8, nv_n = a.ns_cols / 8;
      for (int jg = 0; jg < R / 8; ++jg) {
        const int j = jg * 8 + jl;
        const uint8_t *ar = j < r ? S.arow[j] : nullptr;
        for (int kv = warp * 4 + vo; kv < kv_n; kv += kPfEpiWarps * 4) {
          const uint32_t dst = aw_u + kv * lbo_a + jg * 128 + jl * 16;
          if (j < r && kv * 8 < ks_valid) {
            const uint8_t *src = ar ? ar + kv * 16 : nullptr;
            if (!ar) {
              long long room;
              src = pool_addr(a.pool, slot, a.a_off + ((long long)j * a.d_in + kb0 * kBoxCols + kv * 8) * 2, &room);
              if (!src) {
                set_status(a.status, LORA_ERR_NOT_LOADED);
                src = a.pool.base;
              }
            }
            cp_async16_pf(dst, src);
          } else {
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
          }
        }
        const uint8_t *br = j < r ? S.brow[j] : nullptr;
        for (int nv = warp * 4 + vo; nv < nv_n; nv += kPfEpiWarps * 4) {
          const uint32_t dst = bw_u + jg * lbo_b + nv * 128 + jl * 16;
          if (j < r && nv * 8 < ns_valid) {
            const uint8_t *src = br ? br + nv * 16 : nullptr;
            if (!br) {
              long long room;
              src = pool_addr(a.pool, slot, a.bt_off + ((long long)j * a.d_out + q0 * kChunkCols + nv * 8) * 2,
                              &room);
              if (!src) {
                set_status(a.status, LORA_ERR_NOT_LOADED);
                src = a.pool.base;
              }
            }
            cp_async16_pf(dst, src);
          } else {
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
          }
        }
      }
      cp_async_wait_all();
      fence_async_smem();  // generic-proxy writes -> visible to the MMAs (async proxy)
      pf_arrive(S.w_full);

      // (2) this CTA's share of V (row tid of the tile) out of TMEM
      float vrow[kPfRankCap];
#pragma unroll
      for (int j = 0; j < kPfRankCap; ++j) vrow[j] = 0.f;
      epi_wait(S.sh_done, tpar, a.status, alive);
      tc_fence_after();
      const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
      if (nkb > 0 && alive) {
        float t16[16];
        tmem_ld16(lane_base + kVCol, t16);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) vrow[j] = t16[j];
        if (R > 16) {
          tmem_ld16(lane_base + kVCol + 16, t16);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) vrow[16 + j] = t16[j];
        }
      }
      // (3) sum the shares over the cluster in fixed CTA order: publish the
      // share, signal every peer, read every peer's share, then tell every
      // peer its buffer may be reused
      if (tcount > 0) epi_wait_cluster(S.part_free, (tcount - 1) & 1u, a.status, alive);
#pragma unroll
      for (int j = 0; j < kPfRankCap; ++j)
        if (j < R) S.part[tid * a.r_cap + j] = vrow[j];
      __syncwarp();
      if (lane == 0)
        for (int c = 0; c < C; ++c) mbar_arrive_remote(S.part_ready, (uint32_t)c);
      epi_wait_cluster(S.part_ready, tpar, a.status, alive);
#pragma unroll
      for (int j = 0; j < kPfRankCap; ++j) vrow[j] = 0.f;
      for (int c = 0; c < C; ++c) {
        const float *rp = cluster.map_shared_rank(S.part, c) + tid * a.r_cap;
#pragma unroll
        for (int j = 0; j < kPfRankCap; ++j)
          if (j < R) vrow[j] += rp[j];
      }
      __syncwarp();
      if (lane == 0)
        for (int c = 0; c < C; ++c) mbar_arrive_remote(S.part_free, (uint32_t)c);
      // (4) V as two bf16 MMA operands (hi + lo), K-major core matrices
#pragma unroll
      for (int j8 = 0; j8 < kPfRankCap / 8; ++j8) {
        if (j8 >= R / 8) break;
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
      pf_arrive(S.v_full);

      // (5) expand epilogue: y box (64 columns) by y box, in the ring order
      const float scale = a.scales[slot];
      for (int q = 0; q < nq; ++q) {
        const uint32_t e = ge + q, b = e & 1u;
        epi_wait(&S.ex_done[b], (e >> 1) & 1, a.status, alive);
        tc_fence_after();
        for (int h = 0; h < 2; ++h) {
          const uint32_t g = gbase + nkb + 2 * q + h, st = g % NS;
          epi_wait(&S.full[st], (g / NS) & 1, a.status, alive);
          float acc[64];
          if (alive) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float t16[16];
              tmem_ld16(lane_base + b * kChunkCols + h * kBoxCols + c * 16, t16);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 16; ++k) acc[c * 16 + k] = t16[k];
            }
          }
          // y + s * acc in place, row tid of the box (128-byte swizzle)
          uint8_t *box = S.ring + st * kBoxBytes;
          const int col0 = (q0 + q) * kChunkCols + h * kBoxCols;
          if (alive) {
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {
              uint4 *pv = reinterpret_cast<uint4 *>(box + tid * 128 + ((c16 ^ (tid & 7)) * 16));
              const uint4 u = *pv;
              float yv[8];
              unpack8(u, yv);
              uint4 o;
              o.x = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 0], yv[0]), fmaf(scale, acc[c16 * 8 + 1], yv[1]));
              o.y = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 2], yv[2]), fmaf(scale, acc[c16 * 8 + 3], yv[3]));
              o.z = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 4], yv[4]), fmaf(scale, acc[c16 * 8 + 5], yv[5]));
              o.w = pack_bf16x2(fmaf(scale, acc[c16 * 8 + 6], yv[6]), fmaf(scale, acc[c16 * 8 + 7], yv[7]));
              *pv = o;
            }
          }
          __syncwarp();
          // this warp's 32 rows out, 8 lanes per 128-byte row; only the
          // tile's own rows and columns inside d_out
          if (alive) {
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int rl = warp * 32 + it * 4 + (lane >> 3), c = lane & 7;
              const int col = col0 + c * 8;
              if (rl < m && col < a.d_out) {
                const uint4 v = *reinterpret_cast<const uint4 *>(box + rl * 128 + ((c ^ (rl & 7)) * 16));
                *reinterpret_cast<uint4 *>(a.y + (long long)(row0 + rl) * a.ldy + col) = v;
              }
            }
          }
          epi_sync();  // every epilogue warp is done with the box
          if (tid == 0) pf_arrive(&S.empty[st]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) pf_arrive(&S.ex_free[b]);
      }
    }
    gbase += nkb + n_ybox;
    ge += nq;
    ++tcount;
  }

  // no CTA leaves while a peer may still arrive on or read its shared memory
  tc_fence_before();
  __syncthreads();
  cluster.sync();
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

// Pick the cluster size and ring depth that fit shared memory; false if the
// tensor-core path cannot serve this target (the decode kernel then takes the
// long segments too).  Few tiles (bounded by max_tiles) favour 8-CTA
// clusters, so that more SMs share each tile.
bool prefill_geometry(const lora_pool *pool, int target, int max_tiles, PrefillGeometry *g) {
  if (pool->r_max > kPfRankCap) return false;
  const int d_in = pool->targets[target].d_in, d_out = pool->targets[target].d_out;
  const int r_cap = pool->r_max <= 16 ? 16 : 32;
  const int nkb_all = (d_in + kBoxCols - 1) / kBoxCols, nq_all = (d_out + kChunkCols - 1) / kChunkCols;
  const int cap = 227 * 1024;
  const int order_many[2] = {4, 8}, order_few[2] = {8, 4};
  const int *order = (long long)max_tiles * 4 >= 148 ? order_many : order_few;
  for (int want : {6, 2}) {
    for (int oi = 0; oi < 2; ++oi) {
      const int C = order[oi];
      const int ks = ((nkb_all + C - 1) / C) * kBoxCols, ns = ((nq_all + C - 1) / C) * kChunkCols;
      for (int st = kPfMaxStages; st >= want; --st) {
        const int smem = pf_smem_bytes(st, r_cap, ks, ns);
        if (smem <= cap) {
          *g = {C, st, r_cap, ks, ns, smem};
          return true;
        }
      }
    }
  }
  return false;
}

int launch_prefill(lora_pool *pool, int target, const void *x, int ldx, void *y, int ldy, const float *scales,
                   int T, const void *ws, cudaStream_t st) {
  PlanLayout L = plan_layout(T);
  PrefillGeometry geo;
  if (!prefill_geometry(pool, target, L.j_max, &geo)) return LORA_ERR_INVALID_ARG;
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
  a.n_stages = geo.n_stages;

  static int attr_smem[64] = {};
  if (pool->device < 0 || pool->device >= 64) return LORA_ERR_INVALID_ARG;
  if (attr_smem[pool->device] < geo.smem) {
    if (cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
        cudaSuccess)
      return LORA_ERR_CUDA;
    attr_smem[pool->device] = 227 * 1024;
  }
  cudaLaunchConfig_t cfg = {};
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
  // one wave of co-resident clusters; they loop over the tiles
  // (tiles <= T / 128 + number of long segments)
  int fit = 0;
  {
    std::lock_guard<std::mutex> lk(pool->mu);
    auto key = std::make_pair(geo.C, geo.smem);
    auto it = pool->prefill_fit.find(key);
    if (it != pool->prefill_fit.end()) {
      fit = it->second;
    } else {
      cfg.gridDim = dim3(geo.C);
      if (cudaOccupancyMaxActiveClusters(&fit, prefill_kernel, &cfg) != cudaSuccess || fit < 1) {
        (void)cudaGetLastError();
        return LORA_ERR_CUDA;
      }
      pool->prefill_fit[key] = fit;
    }
  }
  const int n_clusters = std::max(1, std::min(L.j_max, fit));
  cfg.gridDim = dim3(n_clusters * geo.C);
  g_launches.fetch_add(1);
  if (cudaLaunchKernelEx(&cfg, prefill_kernel, a) != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

}  // namespace lora
