// internal.cuh -- shared definitions of the B200 multi-LoRA delta library.
//
// Device-side views of the adapter pool and of a batch plan, the plan layout
// inside the caller's workspace, and the handful of sm_100a PTX wrappers the
// kernels use (mbarriers, 1-D bulk async copies, grid-dependency control,
// bounded waits).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <map>
#include <mutex>
#include <unordered_map>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "lora.h"

namespace lora {

// A named NVTX range over one C-ABI call (host side: seen by profilers that
// record NVTX ranges, a few nanoseconds otherwise).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

// ---------------------------------------------------------------- limits
constexpr int kRMax = 64;            // largest slot rank
constexpr int kMaxSlots = 16384;     // plan kernel keeps one counter per slot in smem
constexpr int kMaxTargets = 4096;
constexpr int kMaxTokens = 1 << 20;
constexpr int kItemRows = 16;        // rows per decode work item

constexpr int kMmaRows = 128;        // rows per tensor-core tile
constexpr int kMmaMinRows = 64;     // segment length that selects the tensor-core path
constexpr int kPlanThreads = 1024;
constexpr int kConsumerWarps = 8;    // decode kernel: 8 compute warps (plus one producer warp)
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kMaxStages = 4;        // barrier slots of the decode ring (it runs n_stages <= this)
constexpr int kFusedMaxT = 256;      // batches up to this size are grouped inside the decode kernel
constexpr int kMaxMulti = 4;         // targets sharing x in one decode launch

extern std::atomic<uint64_t> g_launches;

// ---------------------------------------------------------------- views
struct PoolView {
  const uint8_t *base;     // page memory
  const int32_t *pt;       // [n_slots][pps] physical page, -1 = none
  const int32_t *rank;     // [n_slots][n_targets] rank of the adapter on a target
  const int32_t *loaded;   // [n_slots] 1 = slot holds pages
  long long page_bytes;
  int pps;                 // pages per slot
  int log2_page;           // -1: one page per slot
  int n_slots;
  int n_targets;
  int n_pages;             // physical pages of the pool memory
};

// LORA_DEBUG builds check each index, page and byte range before it is used
// for a load, a copy or a store; dbg_ok() records LORA_ERR_BOUNDS in the
// sticky status and returns false where a check fails (the caller then skips
// or redirects the access).  Other builds compile the checks away.
#ifdef LORA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool dbg_ok(bool ok, int *status) {
  if (!kDebugChecks) return true;
  if (!ok) atomicCAS(status, 0, LORA_ERR_BOUNDS);
  return ok;
}
// LORA_DEBUG: the slot range [off, off + bytes) of a slot lies inside the
// slot, and each page it touches inside the pool memory.
__device__ __forceinline__ bool dbg_slot_range(const PoolView &p, int slot, long long off, long long bytes,
                                               int *status) {
  if (!kDebugChecks) return true;
  const long long slot_bytes = p.log2_page < 0 ? p.page_bytes : (long long)p.pps * p.page_bytes;
  return dbg_ok(slot >= 0 && slot < p.n_slots && off >= 0 && bytes >= 0 && off + bytes <= slot_bytes, status);
}

// Physical address of logical byte `off` of `slot`, and how many bytes stay
// on the same page from there.
__device__ __forceinline__ const uint8_t *pool_addr(const PoolView &p, int slot,
                                                    long long off, long long *room) {
  long long page_idx, inside;
  if (p.log2_page < 0) {
    page_idx = 0;
    inside = off;
    *room = p.page_bytes - off;
  } else {
    page_idx = off >> p.log2_page;
    inside = off & (p.page_bytes - 1);
    *room = p.page_bytes - inside;
  }
  int phys = __ldg(p.pt + (long long)slot * p.pps + page_idx);
  if (phys < 0) return nullptr;
  return p.base + (long long)phys * p.page_bytes + inside;
}

// Physical page holding a slot's whole block [first, first + bytes), or -1
// when the block spans pages (its pieces are then located one by one).
__device__ __forceinline__ int block_page(const PoolView &p, int slot, long long first, long long bytes) {
  if (p.log2_page < 0) return __ldg(p.pt + (long long)slot * p.pps);
  const long long pf = first >> p.log2_page, pl = (first + bytes - 1) >> p.log2_page;
  return pf == pl ? __ldg(p.pt + (long long)slot * p.pps + pf) : -1;
}

// Address of logical byte `off` of a slot whose block lies on physical page
// `page` (block_page >= 0).
__device__ __forceinline__ const uint8_t *page_addr(const PoolView &p, int page, long long off) {
  return p.base + (long long)page * p.page_bytes + (p.log2_page < 0 ? off : (off & (p.page_bytes - 1)));
}

// Arrangement of an adapter block inside a slot.  A block (A: r_max rows of
// d_in bf16; B^T: r_max rows of d_out bf16) is stored in column tiles of
// pool_tile_cols(r_max) columns (32 KiB of r_max rows) -- the tile the decode
// kernel stages with one bulk copy.  Tile k holds columns [k * tc, min((k + 1) * tc, width)) of rows
// 0 .. r_max - 1, one row after the other, so the first r rows of a tile are
// one contiguous range.  Inside a row of a tile, the 16-byte chunks of every
// complete group of eight are permuted, chunk c stored at c ^ (row % 8) (a
// trailing partial group keeps its order): the rows of a staged tile then
// sit in different shared-memory banks for the MMA operand loads.
__host__ __device__ constexpr int pool_tile_cols(int r_max) { return r_max <= 16 ? 1024 : r_max <= 32 ? 512 : 256; }

__host__ __device__ constexpr int swz_chunk(int c, int row, int chunks) {
  return ((c | 7) < chunks) ? (c ^ (row & 7)) : c;
}

// Byte offset, inside a block of `width` columns, of 16-byte chunk `chunk`
// (columns 8 chunk .. 8 chunk + 7) of row `row`.
__host__ __device__ constexpr long long block_chunk_off(int row, int chunk, int width, int r_max) {
  const int tcc = pool_tile_cols(r_max) / 8;  // chunks per full tile
  const int k = chunk / tcc, c = chunk - k * tcc;
  const int rest = width / 8 - k * tcc;
  const int tw = rest < tcc ? rest : tcc;  // chunks in this tile
  return (long long)k * r_max * tcc * 16 + (long long)row * tw * 16 + (long long)swz_chunk(c, row, tw) * 16;
}

// Plan arrays inside the workspace (byte offsets from its base).
struct PlanLayout {
  size_t header, perm, seg_start, seg_slot, seg_row, items, tiles, total;
  int s_max, i_max, j_max;
};

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Segment length from which a segment plan uses the tensor cores: a batch of
// few segments (a prefill batch) sends every segment there, so that it needs
// no decode launch for its short segments (a segment of m rows is one tile
// of m rows: its adapter slices and rows are the same bytes either way);
// otherwise segments of kMmaMinRows rows or more.  The few-segment rule
// applies while the tiles stay within the plan's tile capacity.
constexpr int kFewSegments = 16;

constexpr PlanLayout plan_layout(int T) {
  PlanLayout L{};
  const int t = T > 0 ? T : 1;
  L.s_max = t;
  L.i_max = t + (t + kItemRows - 1) / kItemRows;
  L.j_max = (3 * t + kMmaRows - 1) / kMmaRows + 1;
  size_t off = 0;
  L.header = off;    off = align256(off + 64 * 4);
  L.perm = off;      off = align256(off + size_t(t) * 4);
  L.seg_start = off; off = align256(off + size_t(L.s_max + 1) * 4);
  L.seg_slot = off;  off = align256(off + size_t(L.s_max) * 4);
  L.seg_row = off;   off = align256(off + size_t(L.s_max) * 4);
  L.items = off;     off = align256(off + size_t(L.i_max) * 16);
  L.tiles = off;     off = align256(off + size_t(L.j_max) * 16);
  L.total = off;
  return L;
}

constexpr int segment_mma_min(int S, int T) {
  return (S <= kFewSegments && T / kMmaRows + S <= plan_layout(T).j_max) ? 1 : kMmaMinRows;
}

// Header words of a plan.
// kHdrItemsAll counts the decode items of every segment, long ones included
// (they follow the short segments' items), for targets the tensor-core path
// cannot serve.
enum { kHdrSegs = 0, kHdrActive = 1, kHdrItems = 2, kHdrTiles = 3, kHdrT = 4, kHdrItemsAll = 5 };

struct PlanView {
  int32_t *hdr;
  int32_t *perm;
  int32_t *seg_start;
  int32_t *seg_slot;
  int32_t *seg_row;
  int4 *items;   // {slot, first perm index, rows, segment}
  int4 *tiles;   // {slot, first row, rows, segment}
};

inline PlanView plan_view(void *ws, const PlanLayout &L) {
  uint8_t *b = static_cast<uint8_t *>(ws);
  PlanView v;
  v.hdr = reinterpret_cast<int32_t *>(b + L.header);
  v.perm = reinterpret_cast<int32_t *>(b + L.perm);
  v.seg_start = reinterpret_cast<int32_t *>(b + L.seg_start);
  v.seg_slot = reinterpret_cast<int32_t *>(b + L.seg_slot);
  v.seg_row = reinterpret_cast<int32_t *>(b + L.seg_row);
  v.items = reinterpret_cast<int4 *>(b + L.items);
  v.tiles = reinterpret_cast<int4 *>(b + L.tiles);
  return v;
}

// ---------------------------------------------------------------- PTX
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Test a phase of an mbarrier; while it is incomplete the thread is
// suspended in hardware (it issues nothing) until the phase completes or
// about kSuspendNs pass.  Waiting warps thus leave the SM's issue slots to
// the warps that have work.
constexpr uint32_t kSuspendNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Wait for an mbarrier phase with an iteration cap and a time cap (limit_ns,
// 1 s unless the library's wait limit was lowered).  The time is counted in
// SM clock cycles (clock64, a register read: the global timer costs far more
// per read), two per nanosecond, which is at least limit_ns at any SM clock
// up to 2 GHz.  On giving up, records LORA_ERR_TIMEOUT in the sticky status
// and returns false; the caller skips the work that needed the data.
constexpr uint32_t kSpinLimit = 1u << 22;
constexpr uint64_t kSpinNs = 1000000000ull;

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, int *status,
                                                  uint64_t limit_ns = kSpinNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64(), lim = (long long)(2 * limit_ns);
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > lim) break;
  }
  atomicCAS(status, 0, LORA_ERR_TIMEOUT);
  return false;
}

// Global-memory counters shared by the CTAs of one launch: an add with
// release semantics (the adder's earlier writes become visible first) and a
// load with acquire semantics, both at GPU scope.
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Wait until *p == want, bounded like mbar_wait_bounded.
__device__ __forceinline__ bool wait_count_bounded(const unsigned *p, unsigned want, int *status,
                                                   uint64_t limit_ns = kSpinNs) {
  if (ld_acquire(p) == want) return true;
  const long long t0 = clock64(), lim = (long long)(2 * limit_ns);
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    __nanosleep(64);  // (a poll is a global round trip; the sleep keeps the warp off the issue slots)
    if (ld_acquire(p) == want) return true;
    if (clock64() - t0 > lim) break;
  }
  atomicCAS(status, 0, LORA_ERR_TIMEOUT);
  return false;
}

// 1-D bulk async copy global -> this CTA's shared memory, completing on an
// mbarrier (no multicast).  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 1-D bulk async copy this CTA's shared memory -> global, in the issuing
// thread's current bulk group.  dst, src 16-byte aligned; bytes a multiple of
// 16.  The source may be reused once bulk_wait_read() returns; the data are
// in global memory once bulk_wait_all() returns.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// The same, for all but the newest bulk group.
__device__ __forceinline__ void bulk_wait_read_but_newest() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Hint: start bringing `bytes` at src into L2 (nothing is returned or waited
// for).  src 16-byte aligned, inside a live allocation; bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// The GPU's global nanosecond timer.
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch: wait for the grids this one depends on.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// bf16 pair <-> fp32 (exact decode; round-to-nearest-even encode).
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ void unpack8(const uint4 &u, float f[8]) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
  f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z);
  f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void set_status(int *status, int code) { atomicCAS(status, 0, code); }

// LORA_DEBUG: `bytes` from the pool's first page(s) instead of a range that
// failed its check, so that the bytes a stage expects still arrive.
__device__ __forceinline__ void bulk_g2s_redirect(uint8_t *dst, const PoolView &pool, uint32_t bytes,
                                                  uint64_t *bar) {
  while (bytes > 0) {
    const uint32_t n = (uint32_t)min((long long)bytes, pool.page_bytes);
    bulk_g2s(dst, pool.base, n, bar);
    dst += n;
    bytes -= n;
  }
}
// LORA_DEBUG: `bytes` from logical byte `off` of a block on physical page
// `page` stay inside that page and the page inside the pool memory.
__device__ __forceinline__ bool dbg_page_range(const PoolView &p, int page, long long off, long long bytes,
                                               int *status) {
  if (!kDebugChecks) return true;
  const long long inside = p.log2_page < 0 ? off : (off & (p.page_bytes - 1));
  return dbg_ok(page >= 0 && page < p.n_pages && inside >= 0 && inside + bytes <= p.page_bytes, status);
}

// Copy `bytes` of slot's logical range starting at `off` into dst, cut at
// page boundaries.  A missing page (slot unloaded under our feet) is replaced
// by page-free reads of the pool base and reported.
__device__ __forceinline__ void copy_pool_row(const PoolView &pool, int slot, long long off, uint32_t bytes,
                                              uint8_t *dst, uint64_t *bar, int *status) {
  if (!dbg_slot_range(pool, slot, off, bytes, status)) {
    bulk_g2s_redirect(dst, pool, bytes, bar);
    return;
  }
  while (bytes > 0) {
    long long room;
    const uint8_t *src = pool_addr(pool, slot, off, &room);
    uint32_t n = (uint32_t)min((long long)bytes, room);
    if (src == nullptr) {
      set_status(status, LORA_ERR_NOT_LOADED);
      src = pool.base;
    }
    if (kDebugChecks && src != pool.base &&
        !dbg_ok(src >= pool.base && src + n <= pool.base + (long long)pool.n_pages * pool.page_bytes, status))
      src = pool.base;
    bulk_g2s(dst, src, n, bar);
    dst += n;
    off += n;
    bytes -= n;
  }
}


// Launch attribute for programmatic dependent launch: the kernel may start
// while the previous kernel on the stream is still running; it reads that
// kernel's results only after griddep_wait().  Kernels of this library call
// griddep_launch_dependents() once they have passed their own griddep_wait(),
// so a kernel that starts early knows that everything before its
// predecessor has completed.
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute at;
  at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at.val.programmaticStreamSerializationAllowed = 1;
  return at;
}

}  // namespace lora

// ---------------------------------------------------------------- host pool
struct lora_pool {
  int device = 0;
  int n_targets = 0, r_max = 0, n_slots = 0;
  std::vector<lora_target> targets;
  std::vector<long long> a_off, bt_off;
  long long slot_bytes = 0;
  long long page_bytes = 0;
  int pps = 0, log2_page = -1;
  int n_pages = 0;
  uint8_t *mem = nullptr;
  size_t mem_bytes = 0;
  std::vector<int32_t> free_pages;  // stack; back() is handed out next
  std::vector<int32_t> pt, rank, loaded;
  void *dev_tables = nullptr;
  int32_t *d_pt = nullptr, *d_rank = nullptr, *d_loaded = nullptr;
  int *d_status = nullptr;
  int decode_per_sm = 0;    // co-resident decode CTAs per SM at this pool's r_max
  int decode_max_ctas = 0;  // and on the whole device
  // Kind of the plan last built into each workspace (1 = index vector,
  // 2 = segments, which may hold tensor-core tiles); kept on the host so that
  // an apply call can pick its kernels without reading the device.
  std::unordered_map<const void *, int> plan_kind;
  std::map<std::pair<int, int>, int> prefill_fit;  // (kernel, smem) -> co-resident CTAs
  std::mutex mu;

  lora::PoolView view() const {
    lora::PoolView v;
    v.base = mem;
    v.pt = d_pt;
    v.rank = d_rank;
    v.loaded = d_loaded;
    v.page_bytes = page_bytes;
    v.pps = pps;
    v.log2_page = log2_page;
    v.n_slots = n_slots;
    v.n_targets = n_targets;
    v.n_pages = n_pages;
    return v;
  }
};

namespace lora {

// Makes the pool's device current for the scope of a call.
struct DeviceGuard {
  int prev = -1, want = -1;
  explicit DeviceGuard(int d) : want(d) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != d) cudaSetDevice(d);
  }
  ~DeviceGuard() {
    if (prev >= 0 && prev != want) cudaSetDevice(prev);
  }
};

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launchers (defined in plan.cu / decode.cu).
int launch_plan_ids(lora_pool *pool, const int32_t *ids, int T, void *ws, cudaStream_t st);
int launch_plan_segments(lora_pool *pool, const int32_t *off, const int32_t *slot, int S, int T,
                         void *ws, cudaStream_t st);
enum DecodeMode { kFused = 0, kShrinkOnly = 1, kExpandOnly = 2 };
// One decode launch (decode.cu).  ids != nullptr: the kernel groups ids[0 ..
// T) itself (T <= kFusedMaxT); else it reads the plan in ws (items counted by
// header word items_hdr).  Targets share x,
// d_in and d_out; target i writes columns y_cols[i] .. + d_out - 1 of y.
// Routed expert pairs: x_div = top_k (row p reads x row p / top_k) and, for
// in-kernel grouping, moe_topk / moe_k / moe_e form the pairs' slots.
struct DecodeCall {
  int mode = kFused;
  int n_tgt = 1;
  const int *targets = nullptr;
  const int *y_cols = nullptr;
  const void *x = nullptr;
  int ldx = 0;
  void *y = nullptr;
  int ldy = 0;
  const float *scales = nullptr;
  float *v = nullptr;  // shrink-only output / expand-only input, [T, ldv] fp32
  int ldv = 0;
  int T = 0;
  void *ws = nullptr;  // the plan (plan path only)
  const int32_t *ids = nullptr;
  int items_hdr = kHdrItems;
  int x_div = 1;
  const int32_t *moe_topk = nullptr;
  int moe_k = 0, moe_e = 0;
  int stall = 0;  // test only: the producer fills no stage, so every consumer wait runs out
};
int launch_decode(lora_pool *pool, const DecodeCall &c, cudaStream_t st);
// Lowers (ns > 0) or restores (0) the wall-clock limit of the decode
// kernel's bounded waits; 1 s by default.
void set_wait_limit_ns(unsigned long long ns);
// Writes each routed pair's slot (as the in-kernel grouping forms it) to pair_ids.
int launch_moe_pair_ids(const lora_pool *pool, const int32_t *lora_ids, const int32_t *topk, int n_pairs,
                        int top_k, int n_experts, int32_t *pair_ids, cudaStream_t st);
struct PrefillGeometry {
  int r_cap, kb_per, n_ks, n_stages, n_groups, smem_sh, smem_ex;
};
bool prefill_geometry(const lora_pool *pool, int target, int max_tiles, PrefillGeometry *g);
// Workspace bytes the segment path needs after the plan (fp32 partial V of
// every k-slice); 0 when the tensor-core path cannot serve the target.
size_t prefill_scratch_bytes(const lora_pool *pool, int target, int T);
int launch_prefill(lora_pool *pool, int target, const void *x, int ldx, void *y, int ldy, const float *scales,
                   int T, const void *ws, size_t ws_bytes, cudaStream_t st);
int decode_setup(lora_pool *pool);
// Base projection fused with the delta (linear.cu): y = W x + s_a B_a v, v the
// shrink's fp32 output [T, ldv].
int launch_linear(lora_pool *pool, int target, const void *x, int ldx, const void *W, int ldw, void *y, int ldy,
                  const int32_t *ids, const float *scales, const float *v, int ldv, int T, cudaStream_t st);

}  // namespace lora
