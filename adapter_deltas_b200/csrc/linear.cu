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
// dependent (only the delta waits for v; the W stream may start while the
// shrink still runs, where an SM has room for both):
//   tile     = 128 output features (MMA M) x NT rows of the batch (MMA N).
//              The features are the A operand (W rows, K-major), so a decode
//              batch of 16 .. 256 rows is the N of a single MMA.
//   cluster  = `split` CTAs sharing a tile, each over a K range of d_in:
//                D[f, t]  = sum_k W[f, k] x[t, k]            (TMA, 128 B swizzle)
//              then, as further K steps of the same TMEM accumulator, its
//              share of the tile's adapters (adapter index mod split):
//                D[f, t] += sum_j B_a^T[j, f] (s_a v[t, j])  (rows of adapter a only)
//              with s_a v split into two bf16 terms (hi + lo, ~16 bits kept),
//              16 ranks per chunk, chunks resident in shared memory in groups
//              (the first group's B^T slices load during the W stream).
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
constexpr int kLnMaxChunks = 16;                         // delta chunks resident at once
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
  int n_slots_d;        // delta chunks resident at once (one group)
  int v_cols;           // columns of v staged per row (the pool's r_max); 0: v read in place
  uint32_t tmem_cols;
};

struct LnSmem {
  uint8_t *ring;        // n_stages x (W box | x box)
  float *recv;          // [split][128 / split][nt + 4] partials, over the ring once it is idle
  uint8_t *bt, *vv;     // one group of delta chunks: B^T, and V (hi | lo)
  int *row_slot;        // [256] slot of each row of the tile, -1: no delta
  int *tok;             // [256] index of the row's adapter in the tile's list, -1: none
  int *list;            // [256] slot of each adapter of the tile, by first row
  int *lrank;           // [256] its rank on the target
  float *lscale;        // [256] its scale
  int *lpage;           // [256] physical page of its whole B^T block (-1: the block spans pages)
  int *gch;             // [n_slots_d] the group's chunks: adapter index << 8 | first rank row
  float *vst;           // [nt][v_cols] v of the tile's rows
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
__host__ __device__ inline int ln_chunk_bytes(int nt) { return kLnBtBytes + ln_vv_bytes(nt); }
__host__ __device__ inline int ln_fixed_bytes(int nd) {
  return 1024 /* alignment slack */ + 6 * kLnMaxNT * 4 + ((nd * 4 + 15) & ~15) + 8 * 4 + 4 * 4 +
         (2 * kLnMaxStages + 6) * 8 + 16;
}
__host__ __device__ inline int ln_vst_bytes(int nt, int v_cols) { return (nt * v_cols * 4 + 15) & ~15; }
__host__ __device__ inline int ln_smem_bytes(int nt, int ns, int nd, int v_cols) {
  return ln_fixed_bytes(nd) + ln_ring_bytes(nt, ns) + nd * ln_chunk_bytes(nt) + ln_vst_bytes(nt, v_cols);
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
    S.bt = p; p += a.n_slots_d * kLnBtBytes;
    S.vv = p; p += a.n_slots_d * vv_bytes;
    S.vst = reinterpret_cast<float *>(p); p += ln_vst_bytes(NT, a.v_cols);
    S.row_slot = reinterpret_cast<int *>(p); p += kLnMaxNT * 4;
    S.tok = reinterpret_cast<int *>(p); p += kLnMaxNT * 4;
    S.list = reinterpret_cast<int *>(p); p += kLnMaxNT * 4;
    S.lrank = reinterpret_cast<int *>(p); p += kLnMaxNT * 4;
    S.lscale = reinterpret_cast<float *>(p); p += kLnMaxNT * 4;
    S.lpage = reinterpret_cast<int *>(p); p += kLnMaxNT * 4;
    S.gch = reinterpret_cast<int *>(p); p += (a.n_slots_d * 4 + 15) & ~15;
    S.ballot = reinterpret_cast<uint32_t *>(p); p += 8 * 4;
    S.meta = reinterpret_cast<int *>(p); p += 4 * 4;
    // mbarriers need 8-byte alignment: the offset here is a multiple of 16
    uint64_t *b = reinterpret_cast<uint64_t *>(p);
    S.full = b; b += kLnMaxStages;
    S.empty = b; b += kLnMaxStages;
    S.dfull = b; b += 1;
    S.dfree = b; b += 1;
    b += 2;
    S.acc_done = b++;
    S.meta_bar = b++;
    S.tmem_slot = reinterpret_cast<uint32_t *>(b);
  }
  // The builders' rows: adapter, rank and scale, loaded before anything
  // else (ids, the pool tables and the scales were complete before the
  // shrink let this grid start).
  constexpr int kRowsPer = kLnMaxNT / kLnBuilders;
  int r_slot[kRowsPer], r_rank[kRowsPer], r_page[kRowsPer];
  float r_scale[kRowsPer];
  if (warp < 4) {
    int id[kRowsPer];
#pragma unroll
    for (int q = 0; q < kRowsPer; ++q) {
      const int i = tid + q * kLnBuilders;
      id[q] = (i < NT && t0 + i < a.T) ? a.ids[t0 + i] : -1;
    }
#pragma unroll
    for (int q = 0; q < kRowsPer; ++q) {
      const bool in = id[q] >= 0 && id[q] < a.pool.n_slots;
      const int ld = in ? a.pool.loaded[id[q]] : 0;
      const int r = in ? a.pool.rank[id[q] * a.pool.n_targets + a.target] : 0;
      r_scale[q] = in ? a.scales[id[q]] : 0.f;
      r_page[q] = in ? block_page(a.pool, id[q], a.bt_off, (long long)a.pool_r_max * a.d_out * 2) : -1;
      const bool ok = ld && r > 0 && r <= a.pool_r_max;
      r_slot[q] = ok ? id[q] : -1;
      r_rank[q] = ok ? r : 0;
    }
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(S.tmem_slot)),
                 "r"(a.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // The producer thread initialises the barriers and sends the first ring
  // of W and x loads before the setup barrier (nothing else touches the
  // ring yet, and those stages need no empty-wait).
  const int pre = min(NS, nkb);
  if (tid == kLnBuilders) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tmap_x)) : "memory");
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(S.dfull, kLnBuilders);
    mbar_init(S.dfree, 1);
    mbar_init(S.acc_done, 1);
    mbar_init(S.meta_bar, 1);
    fence_mbar_init();
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&S.full[i], (uint32_t)stage_bytes);
      uint8_t *sp = S.ring + i * stage_bytes;
      tma_load_2d(sp, &a.tmap_w, (kb0 + i) * kLnK, m0, &S.full[i]);
      tma_load_2d(sp + kLnWBox, &a.tmap_x, (kb0 + i) * kLnK, t0, &S.full[i]);
    }
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
      for (int i = pre; i < nkb; ++i) {
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
      // the delta, one resident group of chunks at a time: B^T chunk (A
      // operand, feature-major) x V chunk (K-major), hi then lo
      pf_wait(S.meta_bar, 0, a.status, alive);
      const int nch = alive ? S.meta[0] : 0;
      const int ND = a.n_slots_d;
      const uint32_t idesc_d = idesc_bf16(NT, false, true);
      for (int g = 0; g * ND < nch; ++g) {
        pf_wait(S.dfull, g & 1, a.status, alive);
        tc_fence_after();
        const int n_in = min(ND, nch - g * ND);
        for (int b = 0; b < n_in; ++b) {
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint64_t ad = smem_desc(bt_u + b * kLnBtBytes, kLnBtLbo, 128, 0);
            const uint64_t bd = smem_desc(vv_u + b * vv_bytes + part * 2 * lbo_v, lbo_v, 128, 0);
            if (alive) mma_bf16(tmem, ad, bd, idesc_d, true);
          }
        }
        mma_commit(S.dfree);
      }
      mma_commit(S.acc_done);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ builders
    // (1) slot of each row of the tile
#pragma unroll
    for (int q = 0; q < kRowsPer; ++q) S.row_slot[tid + q * kLnBuilders] = r_slot[q];
    builders_sync();
    // (2) the tile's adapters in order of their first row (with rank and
    // scale), and each row's index in that list
    int first[kRowsPer];
#pragma unroll
    for (int q = 0; q < kRowsPer; ++q) {
      const int i = tid + q * kLnBuilders;
      const int s = r_slot[q];
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
    for (int q = 0; q < kRowsPer; ++q) {
      const int i = tid + q * kLnBuilders, f = first[q];
      int idx = -1;
      if (f >= 0) {
        idx = __popc(S.ballot[f >> 5] & ((1u << (f & 31)) - 1u));
        for (int w = 0; w < (f >> 5); ++w) idx += __popc(S.ballot[w]);
        if (f == i) {
          S.list[idx] = r_slot[q];
          S.lrank[idx] = r_rank[q];
          S.lscale[idx] = r_scale[q];
          S.lpage[idx] = r_page[q];
        }
      }
      S.tok[i] = idx;
    }
    builders_sync();
    // (3) this CTA's delta chunks: adapters ks, ks + split, ..., 16 ranks
    // per chunk, in groups of n_slots_d resident chunks
    const int ND = a.n_slots_d;
    int nch = 0;
    for (int ai = ks; ai < n_ad; ai += SP) nch += (S.lrank[ai] + kLnChunk - 1) / kLnChunk;
    if (tid == 0) {
      S.meta[0] = nch;
      pf_arrive(S.meta_bar);
    }
    const int vstride = a.v_cols;
    // the chunks of group g (adapter index << 8 | first rank row), then the
    // B^T row slices they read, resolved through the page table in parallel
    auto plan_group = [&](int g) {
      if (tid == 0) {
        int c = 0;
        const int c_lo = g * ND, c_hi = min(nch, c_lo + ND);
        for (int ai = ks; ai < n_ad && c < c_hi; ai += SP)
          for (int j0 = 0; j0 < S.lrank[ai] && c < c_hi; j0 += kLnChunk, ++c)
            if (c >= c_lo) S.gch[c - c_lo] = (ai << 8) | j0;
      }
      builders_sync();
      const int n_in = min(ND, nch - g * ND);
      return n_in;
    };
    // B^T rows j0 .. j0 + 15 of the tile's 128 features, feature-major core
    // matrices (8 ranks x 8 features); rows past r_max do not exist, rows
    // past the rank are zero in the pool
    auto load_bt = [&](int n_in) {
      for (int idx = tid; idx < n_in * kLnChunk * (kMmaRows / 8); idx += kLnBuilders) {
        const int b = idx >> 8, q = idx & 255;
        const int jl = q & 7, nv = (q >> 3) & (kMmaRows / 8 - 1), jg = q >> 7;
        const int row = jg * 8 + jl;
        const int ch = S.gch[b];
        const int j = (ch & 255) + row, f = m0 + nv * 8;
        const uint32_t dst = bt_u + b * kLnBtBytes + jg * kLnBtLbo + nv * 128 + jl * 16;
        const uint8_t *src = nullptr;
        if (j < a.pool_r_max && f < a.d_out) {
          const long long off = a.bt_off + block_chunk_off(j, f / 8, a.d_out, a.pool_r_max);
          const int pg = S.lpage[ch >> 8];
          if (pg >= 0) {
            src = page_addr(a.pool, pg, off);
          } else {  // the block spans pages: look this 16-byte piece up
            long long room;
            src = pool_addr(a.pool, S.list[ch >> 8], off, &room);
          }
        }
        if (src)
          cp_async16_pf(dst, src);
        else
          st_shared_zero16(dst);
      }
    };
    // V: s_a v[t, j0 .. j0 + 15] for the rows of the chunk's adapter, zero
    // for the others; K-major core matrices (8 rows x 8 ranks), hi then lo
    auto build_v = [&](int n_in) {
      for (int idx = tid; idx < n_in * 2 * NT; idx += kLnBuilders) {
        const int b = idx / (2 * NT), q = idx - b * 2 * NT;
        const int i = q >> 1, jg = q & 1;
        const int ch = S.gch[b], ai = ch >> 8, j0 = (ch & 255) + jg * 8;
        uint32_t hi[4] = {0u, 0u, 0u, 0u}, lo[4] = {0u, 0u, 0u, 0u};
        if (S.tok[i] == ai) {
          const float sc = S.lscale[ai];
          const int r = S.lrank[ai];
          const float *src = vstride ? S.vst + i * vstride + j0 : a.v + (long long)(t0 + i) * a.ldv + j0;
          float f8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f8[e] = (j0 + e < r) ? sc * src[e] : 0.f;
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
    };
    // (4) the first group's B^T loads leave now, during the W stream; v of
    // the tile's rows is staged once the shrink has finished
    int n_in = nch > 0 ? plan_group(0) : 0;
    load_bt(n_in);
    griddep_wait();
    griddep_launch_dependents();
    if (nch > 0 && vstride > 0) {
      const int rows = min(NT, a.T - t0), n = rows * vstride;
      for (int e0 = 0; e0 < n; e0 += 4 * kLnBuilders) {
        float f[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * kLnBuilders + tid;
          const int i = e / vstride;
          f[u] = (e < n && S.tok[i] >= 0) ? a.v[(long long)(t0 + i) * a.ldv + (e - i * vstride)] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * kLnBuilders + tid;
          if (e < n) S.vst[e] = f[u];
        }
      }
      builders_sync();
    }
    for (int g = 0; g * ND < nch; ++g) {
      if (g > 0) {
        warp_wait(S.dfree, (g - 1) & 1, a.status, alive);  // the previous group's MMAs are done
        n_in = plan_group(g);
        load_bt(n_in);
      }
      build_v(n_in);
      cp_async_wait_all();
      fence_async_smem();  // generic-proxy writes -> visible to the MMAs
      pf_arrive(S.dfull);
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
    for (int c0 = 0; c0 < NT; c0 += 64) {
      float acc[64];
      const int nc = min(64, NT - c0);
#pragma unroll
      for (int h = 0; h < 4; ++h)
        if (h * 16 < nc)
          tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(c0 + 16 * h),
                    *reinterpret_cast<float(*)[16]>(acc + 16 * h));
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q * 4 < nc)
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
// Tiles, cluster size, ring depth and delta chunk groups for a call.
struct LinearGeometry {
  int nt, n_tt, n_mt, split, kb_total, kb_per, n_stages, n_slots_d, v_cols, smem;
  uint32_t tmem_cols;
};

// Stages, chunk slots and v staging within `cap` bytes of shared memory;
// false if not even two stages and two chunks fit.
static bool ln_fit(LinearGeometry &g, int cap, int max_stages, int v_cols) {
  if (ln_fixed_bytes(2) + ln_ring_bytes(g.nt, 2) + ln_vst_bytes(g.nt, v_cols) + 2 * ln_chunk_bytes(g.nt) > cap)
    v_cols = 0;  // v is then read in place
  const int vst = ln_vst_bytes(g.nt, v_cols);
  int ns = std::max(2, std::min(max_stages, g.kb_per));
  while (ns > 2 && ln_fixed_bytes(2) + ln_ring_bytes(g.nt, ns) + vst + 2 * ln_chunk_bytes(g.nt) > cap) --ns;
  int nd = kLnMaxChunks;
  while (nd >= 2 && ln_smem_bytes(g.nt, ns, nd, v_cols) > cap) --nd;
  if (nd < 2) return false;
  g.n_stages = ns;
  g.n_slots_d = nd;
  g.v_cols = v_cols;
  g.smem = ln_smem_bytes(g.nt, ns, nd, v_cols);
  return true;
}

static LinearGeometry linear_geometry(const lora_pool *pool, int T, int d_in, int d_out) {
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
  g.tmem_cols = 32;
  while ((int)g.tmem_cols < g.nt) g.tmem_cols *= 2;
  // W stream depth: about 120 KB of stages for decode-sized tiles, 150 KB
  // for large ones; the rest of the shared memory holds delta chunks (a
  // decode tile's share of adapters usually in one group) and v
  const int budget = g.nt <= 128 ? 120 * 1024 : 150 * 1024;
  const int stages = std::min(kLnMaxStages, std::max(2, budget / ln_stage_bytes(g.nt)));
  if (!ln_fit(g, 227 * 1024, stages, pool->r_max)) g.smem = 227 * 1024 + 1;
  return g;
}

int launch_linear(lora_pool *pool, int target, const void *x, int ldx, const void *W, int ldw, void *y, int ldy,
                  const int32_t *ids, const float *scales, const float *v, int ldv, int T, cudaStream_t st) {
  const int d_in = pool->targets[target].d_in, d_out = pool->targets[target].d_out;
  const LinearGeometry g = linear_geometry(pool, T, d_in, d_out);
  if (g.smem > 227 * 1024 || g.n_slots_d < 2) return LORA_ERR_INVALID_ARG;
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
  a.n_slots_d = g.n_slots_d;
  a.v_cols = g.v_cols;
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
