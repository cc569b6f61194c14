// linear.cu -- a projection layer and its multi-LoRA delta in one output pass.
//
// For a batch whose rows each name an adapter a = ids[t] (or none, -1):
//     y[t] = W x[t] + s_a B_a (A_a x[t])
// the whole layer of "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU",
// section "Why can't you just merge LoRA weights into the base model?"
// (y = xW + (x A_i) B_i alpha/r, the xW term shared by every row), with W
// stored d_out x d_in as in the column form of "Serving Many LoRA Adapters
// From One Base Model", section "How it works".  y is written once: the
// delta joins the base product inside the tensor-core accumulator instead of
// being added to a finished y.
//
// Two launches.  The decode kernel in shrink mode writes v = A_a x[t] (fp32)
// for every adapted row; then this kernel, launched as its programmatic
// dependent (it streams W and x while the shrink still runs, and only the
// delta waits for v):
//   tile     = 128 output features (MMA M) x NT rows of the batch (MMA N).
//              The features are the A operand (W rows, K-major), so a decode
//              batch of 16 .. 256 rows is the N of a single MMA.
//   cluster  = `split` CTAs sharing a tile, each over a K range of d_in:
//                D[f, t]  = sum_k W[f, k] x[t, k]            (TMA, 128 B swizzle)
//              then, as further K steps of the same TMEM accumulator, its
//              share of the tile's adapters (adapter index mod split):
//                D[f, t] += sum_j B_a^T[j, f] (s_a v[t, j])  (rows of adapter a only)
//              with s_a v split into two bf16 terms (hi + lo, ~16 bits kept).
//   epilogue = the split partials meet in the owning CTA's shared memory
//              (DSMEM stores between two cluster barriers), are summed in
//              fixed order and rounded to bf16 once.
// Warps 0-3 build the tile's row table and the delta operands, then run the
// epilogue; warp 4 is the TMA producer; warp 5 issues the MMAs.  Every wait is
// bounded; no load uses cluster multicast.
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "internal.cuh"
#include "tc.cuh"

namespace lora {

constexpr int kLnThreads = 192;
constexpr int kLnBuilders = 128;                         // warps 0-3
constexpr int kLnK = 64;                                 // d_in per stage: one 128-byte swizzled row
constexpr int kLnWBox = kLnK * 2 * kMmaRows;             // W box: 128 features x 64
constexpr int kLnMaxStages = 8;
constexpr int kLnMaxNT = 256;                            // batch rows per tile (MMA N)
constexpr int kLnChunk = 16;                             // rank rows per delta step (MMA K)
constexpr int kLnBtBytes = kLnChunk * kMmaRows * 2;      // B^T chunk: 16 ranks x 128 features
constexpr int kLnBtLbo = (kMmaRows / 8) * 128;           // its k-group stride
constexpr int kLnSms = 148;                              // B200 SM count (grid sizing only)

struct __align__(64) LinearArgs {
  CUtensorMap tmap_w;   // W [d_out, d_in] (leading dimension ldw), box 64 x 128
  CUtensorMap tmap_x;   // x [T, d_in] (leading dimension ldx), box 64 x nt
  PoolView pool;
  int target, d_in, d_out, T;
  long long bt_off;     // B^T block of the target inside a slot
  uint16_t *y;
  long long ldy;
  const int32_t *ids;
  const float *scales;
  const float *v;       // [T, ldv] fp32, written by the shrink
  int ldv;
  int *status;
  int pool_r_max;
  int nt;               // batch rows per tile, multiple of 16
  int n_mt;             // feature tiles
  int split;            // CTAs per tile (cluster size), 1, 2 or 4
  int kb_total;         // 64-wide blocks of d_in
  int kb_per;           // blocks per CTA of a cluster
  int n_stages;
  uint32_t tmem_cols;
};

struct LnSmem {
  uint8_t *ring;        // n_stages x (W box | x box)
  float *recv;          // [split][128 / split][nt + 4] partials, over the ring once it is idle
  uint8_t *bt, *vv;     // two B^T chunks; two V chunks (hi | lo)
  int *row_slot;        // [256] slot of each row of the tile, -1: no delta
  int *tok;             // [256] index of the row's adapter in the tile's list, -1: none
  int *list;            // [256] slot of each adapter of the tile, by first row
  uint32_t *ballot;     // [8] first-row flags
  int *meta;            // [0]: delta chunks of this CTA
  uint64_t *full, *empty, *dfull, *dfree, *acc_done, *meta_bar;
  uint32_t *tmem_slot;
};

__host__ __device__ inline int ln_stage_bytes(int nt) { return kLnWBox + nt * kLnK * 2; }
__host__ __device__ inline int ln_recv_bytes(int nt) { return kMmaRows * (nt + 4) * 4; }
__host__ __device__ inline int ln_vv_bytes(int nt) { return 2 * nt * kLnChunk * 2; }
__host__ __device__ inline int ln_ring_bytes(int nt, int ns) {
  const int ring = ns * ln_stage_bytes(nt), recv = ln_recv_bytes(nt);
  return ring > recv ? ring : recv;
}
__host__ __device__ inline int ln_smem_bytes(int nt, int ns) {
  return 1024 /* alignment slack */ + ln_ring_bytes(nt, ns) + 2 * kLnBtBytes + 2 * ln_vv_bytes(nt) +
         3 * kLnMaxNT * 4 + 8 * 4 + 4 * 4 + (2 * kLnMaxStages + 6) * 8 + 16;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void ln_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t ln_mapa(uint32_t addr, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(cta));
  return r;
}
__device__ __forceinline__ void builders_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kLnBuilders) : "memory"); }

// Slot whose delta row t takes, or -1.  Rows with a bad id or an empty slot
// get none here; the shrink launch reports them in the sticky status.
__device__ __forceinline__ int ln_row_slot(const LinearArgs &a, int t) {
  if (t >= a.T) return -1;
  const int id = a.ids[t];
  if (id < 0 || id >= a.pool.n_slots || !a.pool.loaded[id]) return -1;
  const int r = a.pool.rank[id * a.pool.n_targets + a.target];
  return (r > 0 && r <= a.pool_r_max) ? id : -1;
}

__global__ void __launch_bounds__(kLnThreads, 1) linear_kernel(const __grid_constant__ LinearArgs a) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int SP = a.split, NT = a.nt, NS = a.n_stages;
  const int ks = (int)cluster_ctarank();
  const int tile = (int)cluster_id_x();
  const int mt = tile % a.n_mt, tt = tile / a.n_mt;
  const int m0 = mt * kMmaRows, t0 = tt * NT;
  const int kb0 = ks * a.kb_per;
  const int nkb = max(0, min(a.kb_per, a.kb_total - kb0));
  const int stage_bytes = ln_stage_bytes(NT);
  const int vv_bytes = ln_vv_bytes(NT);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  LnSmem S;
  {
    uint8_t *p = base;
    S.ring = p;
    S.recv = reinterpret_cast<float *>(p);
    p += ln_ring_bytes(NT, NS);
    S.bt = p; p += 2 * kLnBtBytes;
    S.vv = p; p += 2 * vv_bytes;
    S.row_slot = reinterpret_cast<int *>(p); p += kLnMaxNT * 4;
    S.tok = reinterpret_cast<int *>(p); p += kLnMaxNT * 4;
    S.list = reinterpret_cast<int *>(p); p += kLnMaxNT * 4;
    S.ballot = reinterpret_cast<uint32_t *>(p); p += 8 * 4;
    S.meta = reinterpret_cast<int *>(p); p += 4 * 4;
    uint64_t *b = reinterpret_cast<uint64_t *>(p);
    S.full = b; b += kLnMaxStages;
    S.empty = b; b += kLnMaxStages;
    S.dfull = b; b += 2;
    S.dfree = b; b += 2;
    S.acc_done = b++;
    S.meta_bar = b++;
    S.tmem_slot = reinterpret_cast<uint32_t *>(b);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(S.tmem_slot)),
                 "r"(a.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == kLnBuilders) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.dfull[0], kLnBuilders);
    mbar_init(&S.dfull[1], kLnBuilders);
    mbar_init(&S.dfree[0], 1);
    mbar_init(&S.dfree[1], 1);
    mbar_init(S.acc_done, 1);
    mbar_init(S.meta_bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *S.tmem_slot;
  const uint32_t ring_u = smem_u32(S.ring), bt_u = smem_u32(S.bt), vv_u = smem_u32(S.vv);
  const uint32_t lbo_v = (uint32_t)(NT / 8) * 128u;  // k-group stride of a V chunk
  bool alive = true;

  if (warp == 4) {
    // ------------------------------------------------ TMA producer
    // W, x, ids and the pool were complete before the shrink let this grid
    // start; only v (read by the builders) waits for the shrink.
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_w)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_x)) : "memory");
      for (int i = 0; i < nkb; ++i) {
        const int st = i % NS;
        if (i >= NS && !pf_wait(&S.empty[st], ((i / NS) - 1) & 1, a.status, alive)) break;
        mbar_arrive_expect_tx(&S.full[st], (uint32_t)stage_bytes);
        uint8_t *sp = S.ring + st * stage_bytes;
        tma_load_2d(sp, &a.tmap_w, (kb0 + i) * kLnK, m0, &S.full[st]);
        tma_load_2d(sp + kLnWBox, &a.tmap_x, (kb0 + i) * kLnK, t0, &S.full[st]);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(NT, false);
      for (int i = 0; i < nkb; ++i) {
        const int st = i % NS;
        pf_wait(&S.full[st], (i / NS) & 1, a.status, alive);
        tc_fence_after();
        const uint32_t wa = ring_u + st * stage_bytes, xa = wa + kLnWBox;
#pragma unroll
        for (int kk = 0; kk < kLnK / 16; ++kk) {
          const uint64_t ad = smem_desc(wa + kk * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(xa + kk * 32, 16, 1024, 2);
          if (alive) mma_bf16(tmem, ad, bd, idesc, (i | kk) != 0);
        }
        mma_commit(&S.empty[st]);  // the stage is free once these MMAs have read it
      }
      // the delta: B^T chunk (A operand, feature-major) x V chunk (K-major)
      pf_wait(S.meta_bar, 0, a.status, alive);
      const int nch = alive ? S.meta[0] : 0;
      const uint32_t idesc_d = idesc_bf16(NT, false, true);
      for (int c = 0; c < nch; ++c) {
        const int b = c & 1;
        pf_wait(&S.dfull[b], (c >> 1) & 1, a.status, alive);
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint64_t ad = smem_desc(bt_u + b * kLnBtBytes, kLnBtLbo, 128, 0);
          const uint64_t bd = smem_desc(vv_u + b * vv_bytes + part * 2 * lbo_v, lbo_v, 128, 0);
          if (alive) mma_bf16(tmem, ad, bd, idesc_d, true);
        }
        mma_commit(&S.dfree[b]);
      }
      mma_commit(S.acc_done);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ builders
    // (1) slot of each row of the tile
#pragma unroll
    for (int q = 0; q < kLnMaxNT / kLnBuilders; ++q) {
      const int i = tid + q * kLnBuilders;
      S.row_slot[i] = i < NT ? ln_row_slot(a, t0 + i) : -1;
    }
    builders_sync();
    // (2) the tile's adapters in order of their first row, and each row's
    // index in that list
    int first[kLnMaxNT / kLnBuilders];
#pragma unroll
    for (int q = 0; q < kLnMaxNT / kLnBuilders; ++q) {
      const int i = tid + q * kLnBuilders;
      const int s = S.row_slot[i];
      int f = -1;
      if (s >= 0) {
        f = i;
        for (int k = 0; k < i; ++k)
          if (S.row_slot[k] == s) {
            f = k;
            break;
          }
      }
      first[q] = f;
      const uint32_t bal = __ballot_sync(0xffffffffu, s >= 0 && f == i);
      if (lane == 0) S.ballot[warp + 4 * q] = bal;
    }
    builders_sync();
    int n_ad = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) n_ad += __popc(S.ballot[w]);
#pragma unroll
    for (int q = 0; q < kLnMaxNT / kLnBuilders; ++q) {
      const int i = tid + q * kLnBuilders, f = first[q];
      int idx = -1;
      if (f >= 0) {
        idx = __popc(S.ballot[f >> 5] & ((1u << (f & 31)) - 1u));
        for (int w = 0; w < (f >> 5); ++w) idx += __popc(S.ballot[w]);
        if (f == i) S.list[idx] = S.row_slot[i];
      }
      S.tok[i] = idx;
    }
    builders_sync();
    // (3) this CTA's delta steps: adapters ks, ks + split, ..., 16 ranks each
    int nch = 0;
    for (int ai = ks; ai < n_ad; ai += SP) nch += (a.pool.rank[S.list[ai] * a.pool.n_targets + a.target] + 15) >> 4;
    if (tid == 0) {
      S.meta[0] = nch;
      pf_arrive(S.meta_bar);
    }
    // (4) the delta operands, double-buffered against the MMAs
    bool waited = false;
    int c = 0;
    for (int ai = ks; ai < n_ad; ai += SP) {
      const int slot = S.list[ai];
      const int r = a.pool.rank[slot * a.pool.n_targets + a.target];
      const float sc = a.scales[slot];
      for (int j0 = 0; j0 < r; j0 += kLnChunk, ++c) {
        const int b = c & 1;
        if (c >= 2) warp_wait(&S.dfree[b], ((c >> 1) - 1) & 1, a.status, alive);
        // B^T rows j0 .. j0 + 15 of the tile's 128 features, feature-major
        // core matrices (8 ranks x 8 features); rows past r_max do not exist,
        // rows past the rank are zero in the pool
        for (int q = tid; q < kLnChunk * (kMmaRows / 8); q += kLnBuilders) {
          const int jl = q & 7, nv = (q >> 3) & (kMmaRows / 8 - 1), jg = q >> 7;
          const int j = j0 + jg * 8 + jl, f = m0 + nv * 8;
          const uint32_t dst = bt_u + b * kLnBtBytes + jg * kLnBtLbo + nv * 128 + jl * 16;
          const uint8_t *src = nullptr;
          if (j < a.pool_r_max && f < a.d_out) {
            long long room;
            src = pool_addr(a.pool, slot, a.bt_off + ((long long)j * a.d_out + f) * 2, &room);
          }
          if (src)
            cp_async16_pf(dst, src);
          else
            st_shared_zero16(dst);
        }
        if (!waited) {
          griddep_wait();  // v is the shrink's output
          griddep_launch_dependents();
          waited = true;
        }
        // V: s_a v[t, j0 .. j0 + 15] for the rows of this adapter, zero for
        // the others; K-major core matrices (8 rows x 8 ranks), hi then lo
        for (int q = tid; q < 2 * NT; q += kLnBuilders) {
          const int i = q >> 1, jg = q & 1;
          uint32_t hi[4] = {0u, 0u, 0u, 0u}, lo[4] = {0u, 0u, 0u, 0u};
          if (S.tok[i] == ai) {
            const float *src = a.v + (long long)(t0 + i) * a.ldv + j0 + jg * 8;
            float f8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f8[e] = (j0 + jg * 8 + e < r) ? sc * src[e] : 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              hi[e] = pack_bf16x2(f8[2 * e], f8[2 * e + 1]);
              lo[e] = pack_bf16x2(f8[2 * e] - bf16_lo(hi[e]), f8[2 * e + 1] - bf16_hi(hi[e]));
            }
          }
          const uint32_t off = vv_u + b * vv_bytes + jg * lbo_v + (i >> 3) * 128 + (i & 7) * 16;
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(off), "r"(hi[0]), "r"(hi[1]), "r"(hi[2]),
                       "r"(hi[3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(off + 2 * lbo_v), "r"(lo[0]), "r"(lo[1]),
                       "r"(lo[2]), "r"(lo[3])
                       : "memory");
        }
        cp_async_wait_all();
        fence_async_smem();  // generic-proxy writes -> visible to the MMAs
        pf_arrive(&S.dfull[b]);
      }
    }
    if (!waited) {
      griddep_wait();
      griddep_launch_dependents();
    }
    // (5) the accumulator is complete
    warp_wait(S.acc_done, 0, a.status, alive);
    tc_fence_after();
  }

  // Every CTA of the cluster has its accumulator (its builders waited for it
  // before arriving), so every ring is idle: the partials may land there.
  ln_cluster_sync();
  const int per = kMmaRows / SP;  // features each CTA of the cluster writes out
  if (warp < 4) {
    const int owner = (32 * warp) / per;
    const int nloc = 32 * warp - owner * per + lane;
    const uint32_t row = smem_u32(S.recv) + (uint32_t)((ks * per + nloc) * (NT + 4)) * 4u;
    const uint32_t dst = ln_mapa(row, (uint32_t)owner);
    for (int c0 = 0; c0 < NT; c0 += 16) {
      float acc[16];
      tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0, acc);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_cluster_v4(dst + (uint32_t)(c0 + 4 * q) * 4u, acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
    }
  }
  ln_cluster_sync();
  if (warp < 4) {
    // features m0 + ks * per .. + per - 1: partials summed in CTA order
    const int groups = per / 8;
    for (int idx = tid; idx < NT * groups; idx += kLnBuilders) {
      const int i = idx % NT, g = idx / NT;
      const int t = t0 + i, f = m0 + ks * per + g * 8;
      if (t >= a.T || f >= a.d_out) continue;
      float s8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) s8[e] = 0.f;
      for (int src = 0; src < SP; ++src) {
        const float *rp = S.recv + (src * per + g * 8) * (NT + 4) + i;
#pragma unroll
        for (int e = 0; e < 8; ++e) s8[e] += rp[e * (NT + 4)];
      }
      uint4 o;
      o.x = pack_bf16x2(s8[0], s8[1]);
      o.y = pack_bf16x2(s8[2], s8[3]);
      o.z = pack_bf16x2(s8[4], s8[5]);
      o.w = pack_bf16x2(s8[6], s8[7]);
      *reinterpret_cast<uint4 *>(a.y + (long long)t * a.ldy + f) = o;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(a.tmem_cols) : "memory");
  }
}

// ------------------------------------------------------------ host side
// Tiles, cluster size and ring depth for a call.
struct LinearGeometry {
  int nt, n_tt, n_mt, split, kb_total, kb_per, n_stages, smem;
  uint32_t tmem_cols;
};

static LinearGeometry linear_geometry(int T, int d_in, int d_out) {
  LinearGeometry g;
  g.n_tt = (T + kLnMaxNT - 1) / kLnMaxNT;
  const int per_tile = (T + g.n_tt - 1) / g.n_tt;
  g.nt = std::max(16, (per_tile + 15) / 16 * 16);
  g.n_mt = (d_out + kMmaRows - 1) / kMmaRows;
  g.kb_total = (d_in + kLnK - 1) / kLnK;
  const int tiles = g.n_mt * g.n_tt;
  // split d_in over a cluster while the tiles alone leave SMs idle
  g.split = tiles * 4 <= kLnSms + kLnSms / 8 ? 4 : tiles * 2 <= 2 * kLnSms ? 2 : 1;
  while (g.split > 1 && g.split > g.kb_total) g.split /= 2;
  g.kb_per = (g.kb_total + g.split - 1) / g.split;
  while (g.split > 1 && (g.split - 1) * g.kb_per >= g.kb_total) {
    g.split /= 2;
    g.kb_per = (g.kb_total + g.split - 1) / g.split;
  }
  // W stream depth: about 120 KB of stages for decode-sized tiles (room for
  // a shrink CTA beside this one on the SM), 200 KB for large tiles
  const int budget = g.nt <= 128 ? 120 * 1024 : 200 * 1024;
  g.n_stages = std::min(kLnMaxStages, std::max(2, budget / ln_stage_bytes(g.nt)));
  g.n_stages = std::max(2, std::min(g.n_stages, g.kb_per));
  while (g.n_stages > 2 && ln_smem_bytes(g.nt, g.n_stages) > 227 * 1024) --g.n_stages;
  g.smem = ln_smem_bytes(g.nt, g.n_stages);
  g.tmem_cols = 32;
  while ((int)g.tmem_cols < g.nt) g.tmem_cols *= 2;
  return g;
}

int launch_linear(lora_pool *pool, int target, const void *x, int ldx, const void *W, int ldw, void *y, int ldy,
                  const int32_t *ids, const float *scales, const float *v, int ldv, int T, cudaStream_t st) {
  const int d_in = pool->targets[target].d_in, d_out = pool->targets[target].d_out;
  const LinearGeometry g = linear_geometry(T, d_in, d_out);
  if (g.smem > 227 * 1024) return LORA_ERR_INVALID_ARG;
  LinearArgs a;
  memset(&a, 0, sizeof(a));
  if (!make_tmap_2d(&a.tmap_w, W, d_in, d_out, ldw, kLnK, kMmaRows) ||
      !make_tmap_2d(&a.tmap_x, x, d_in, T, ldx, kLnK, g.nt))
    return LORA_ERR_CUDA;
  a.pool = pool->view();
  a.target = target;
  a.d_in = d_in;
  a.d_out = d_out;
  a.T = T;
  a.bt_off = pool->bt_off[target];
  a.y = static_cast<uint16_t *>(y);
  a.ldy = ldy;
  a.ids = ids;
  a.scales = scales;
  a.v = v;
  a.ldv = ldv;
  a.status = pool->d_status;
  a.pool_r_max = pool->r_max;
  a.nt = g.nt;
  a.n_mt = g.n_mt;
  a.split = g.split;
  a.kb_total = g.kb_total;
  a.kb_per = g.kb_per;
  a.n_stages = g.n_stages;
  a.tmem_cols = g.tmem_cols;

  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(linear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  });
  if (attr_err != cudaSuccess) return LORA_ERR_CUDA;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.n_mt * g.n_tt * g.split);
  cfg.blockDim = dim3(kLnThreads);
  cfg.dynamicSmemBytes = g.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = g.split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, linear_kernel, a);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  g_launches.fetch_add(1);
  return LORA_OK;
}

}  // namespace lora
