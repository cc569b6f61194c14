// pool.cu -- the paged adapter pool: slot layout, page free list, page table,
// per-(slot, target) rank table, and the copy of adapter weights into pages.
//
// The pool follows the unified-paging idea of "Multi-LoRA Serving: Sharing One
// GPU Across Adapters" (section "How S-LoRA Proved the Model"): adapter weights
// live in fixed-size pages of one caller-provided buffer, located through a
// page table, so adapters of any rank can come and go without fragmenting
// device memory.  Every slot is padded to the pool's r_max (the static
// max_lora_rank slot of "Multi-LoRA Serving: Why 100 Adapters Fit on One GPU",
// section "Where does multi-LoRA serving actually break?", item 2).
#include <algorithm>
#include <cstring>
#include <new>

#include "internal.cuh"

namespace lora {

std::atomic<uint64_t> g_launches{0};

static bool is_pow2(unsigned long long v) { return v && !(v & (v - 1)); }

// Slot layout: per target an A block (r_max x d_in bf16) then a B^T block
// (r_max x d_out bf16), each starting on a 256-byte boundary.
static long long slot_layout(const lora_target *t, int n, int r_max, std::vector<long long> *a_off,
                             std::vector<long long> *bt_off) {
  long long off = 0;
  for (int i = 0; i < n; ++i) {
    if (a_off) a_off->push_back(off);
    off += (long long)align256(size_t((long long)r_max * t[i].d_in * 2));
    if (bt_off) bt_off->push_back(off);
    off += (long long)align256(size_t((long long)r_max * t[i].d_out * 2));
  }
  return off;
}

static int check_shape(const lora_target *targets, int n_targets, int r_max, int n_slots, size_t page_bytes) {
  if (!targets || n_targets < 1 || n_targets > kMaxTargets) return LORA_ERR_INVALID_ARG;
  if (r_max < 1 || r_max > kRMax) return LORA_ERR_INVALID_ARG;
  if (n_slots < 1 || n_slots > kMaxSlots) return LORA_ERR_INVALID_ARG;
  if (page_bytes != 0 && (!is_pow2(page_bytes) || page_bytes < 4096)) return LORA_ERR_INVALID_ARG;
  for (int i = 0; i < n_targets; ++i) {
    if (targets[i].d_in < 8 || targets[i].d_out < 8) return LORA_ERR_INVALID_ARG;
    if (targets[i].d_in > (1 << 20) || targets[i].d_out > (1 << 20)) return LORA_ERR_INVALID_ARG;
    if ((targets[i].d_in % 8) || (targets[i].d_out % 8)) return LORA_ERR_ALIGNMENT;
  }
  return LORA_OK;
}

// splitmix64, used only to scatter the initial page order.
static uint64_t splitmix64(uint64_t &s) {
  uint64_t z = (s += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Visit the physical pieces of a slot's logical byte range [off, off+bytes).
template <class F>
static void for_each_run(const lora_pool *p, int slot, long long off, long long bytes, F fn) {
  long long done = 0;
  while (done < bytes) {
    long long page_idx = (p->pps == 1) ? 0 : (off + done) / p->page_bytes;
    long long inside = (p->pps == 1) ? (off + done) : (off + done) % p->page_bytes;
    long long n = std::min(bytes - done, p->page_bytes - inside);
    int phys = p->pt[(size_t)slot * p->pps + page_idx];
    fn(p->mem + (long long)phys * p->page_bytes + inside, done, n);
    done += n;
  }
}

// One block of a slot written whole, in the pool's tiled arrangement
// (block_chunk_off): rows below `rank` from src, the rank padding as zeros.
// src is A (rank x width, row-major; transposed = 0) or B (width x rank,
// row-major; transposed = 1, stored as B^T).  One thread per 16-byte chunk.
__global__ void store_block_kernel(PoolView pool, int slot, long long blk_off, int width, int r_max, int rank,
                                   const uint16_t *src, int transposed) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nch = width / 8;
  if (idx >= (long long)nch * r_max) return;
  const int j = (int)(idx / nch), c = (int)(idx % nch);
  uint16_t v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (j < rank) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      v[e] = transposed ? src[(long long)(c * 8 + e) * rank + j] : src[(long long)j * width + c * 8 + e];
  }
  long long room;
  const uint8_t *dst = pool_addr(pool, slot, blk_off + block_chunk_off(j, c, width, r_max), &room);
  if (!dst) return;
  uint4 packed;
  packed.x = v[0] | (uint32_t(v[1]) << 16);
  packed.y = v[2] | (uint32_t(v[3]) << 16);
  packed.z = v[4] | (uint32_t(v[5]) << 16);
  packed.w = v[6] | (uint32_t(v[7]) << 16);
  *reinterpret_cast<uint4 *>(const_cast<uint8_t *>(dst)) = packed;
}

// Host image of one block in the tiled arrangement (see store_block_kernel).
static void block_image(const uint16_t *src, int transposed, int width, int r_max, int rank,
                        std::vector<uint16_t> *img) {
  img->assign((size_t)r_max * width, 0);
  const int nch = width / 8;
  for (int j = 0; j < rank; ++j)
    for (int c = 0; c < nch; ++c) {
      uint16_t *d = img->data() + block_chunk_off(j, c, width, r_max) / 2;
      for (int e = 0; e < 8; ++e)
        d[e] = transposed ? src[(size_t)(c * 8 + e) * rank + j] : src[(size_t)j * width + c * 8 + e];
    }
}

// One target's part of a swap-in: where its A (then its B) sits in the
// staging data and where the target's blocks lie in a slot.
struct SwapDesc {
  long long src, a_off, bt_off, pad;
  int d_in, d_out, rank, pad2;
};
static_assert(sizeof(SwapDesc) == 48, "descriptor layout");

// Staged adapter -> one slot's pages: block y handles target y; its threads
// walk the target's A block (r_max x d_in) then its B^T block (r_max x d_out)
// in 16-byte chunks -- rows below the rank from the staged A and (transposed)
// B, the padding rows as zeros -- and store each through the page table.
__global__ void swap_in_kernel(PoolView pool, int slot, int r_max, const SwapDesc *desc, const uint8_t *data) {
  const SwapDesc d = desc[blockIdx.y];
  const long long per_a = d.d_in / 8, per_b = d.d_out / 8;
  const long long na = (long long)r_max * per_a, nb = (long long)r_max * per_b;
  const uint16_t *B = reinterpret_cast<const uint16_t *>(data + d.src + (long long)d.rank * d.d_in * 2);
  for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < na + nb;
       c += (long long)gridDim.x * blockDim.x) {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    long long off;
    if (c < na) {
      const int j = (int)(c / per_a);
      off = d.a_off + block_chunk_off(j, (int)(c % per_a), d.d_in, r_max);
      if (j < d.rank) v = *reinterpret_cast<const uint4 *>(data + d.src + c * 16);
    } else {
      const long long cb = c - na;
      const int j = (int)(cb / per_b), n0 = (int)(cb % per_b) * 8;
      off = d.bt_off + block_chunk_off(j, (int)(cb % per_b), d.d_out, r_max);
      if (j < d.rank) {
        uint16_t e[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) e[q] = B[(long long)(n0 + q) * d.rank + j];
        v.x = e[0] | (uint32_t(e[1]) << 16);
        v.y = e[2] | (uint32_t(e[3]) << 16);
        v.z = e[4] | (uint32_t(e[5]) << 16);
        v.w = e[6] | (uint32_t(e[7]) << 16);
      }
    }
    long long room;
    const uint8_t *dst = pool_addr(pool, slot, off, &room);
    if (dst) *reinterpret_cast<uint4 *>(const_cast<uint8_t *>(dst)) = v;
  }
}

}  // namespace lora

using namespace lora;

namespace {

// Bytes of a packed swap-in source: for each target with rank > 0, A [rank,
// d_in] then B [d_out, rank], bf16.  -1 for an invalid rank.
long long swap_src_bytes(const lora_pool *p, const int *ranks) {
  long long n = 0;
  for (int t = 0; t < p->n_targets; ++t) {
    if (ranks[t] < 0 || ranks[t] > p->r_max) return -1;
    n += (long long)ranks[t] * (p->targets[t].d_in + p->targets[t].d_out) * 2;
  }
  return n;
}

size_t swap_desc_bytes(const lora_pool *p) { return align256(size_t(p->n_targets) * sizeof(SwapDesc)); }

}  // namespace

#define CUDA_TRY(expr)                            \
  do {                                            \
    if ((expr) != cudaSuccess) {                  \
      (void)cudaGetLastError();                   \
      return LORA_ERR_CUDA;                       \
    }                                             \
  } while (0)

extern "C" {

const char *lora_status_string(int s) {
  switch (s) {
    case LORA_OK: return "LORA_OK";
    case LORA_ERR_INVALID_ARG: return "LORA_ERR_INVALID_ARG";
    case LORA_ERR_ALIGNMENT: return "LORA_ERR_ALIGNMENT";
    case LORA_ERR_NO_PAGES: return "LORA_ERR_NO_PAGES";
    case LORA_ERR_SLOT: return "LORA_ERR_SLOT";
    case LORA_ERR_NOT_LOADED: return "LORA_ERR_NOT_LOADED";
    case LORA_ERR_CUDA: return "LORA_ERR_CUDA";
    case LORA_ERR_BAD_ID: return "LORA_ERR_BAD_ID";
    case LORA_ERR_TIMEOUT: return "LORA_ERR_TIMEOUT";
    case LORA_ERR_WORKSPACE: return "LORA_ERR_WORKSPACE";
    case LORA_ERR_BOUNDS: return "LORA_ERR_BOUNDS";
    default: return "LORA_ERR_UNKNOWN";
  }
}

size_t lora_pool_bytes_required(const lora_target *targets, int n_targets, int r_max, int n_slots,
                                size_t page_bytes) {
  if (check_shape(targets, n_targets, r_max, n_slots, page_bytes) != LORA_OK) return 0;
  long long slot = slot_layout(targets, n_targets, r_max, nullptr, nullptr);
  if (page_bytes == 0) return size_t(n_slots) * align256(size_t(slot));
  long long pps = (slot + (long long)page_bytes - 1) / (long long)page_bytes;
  return size_t(n_slots) * size_t(pps) * page_bytes;
}

int lora_pool_create(lora_pool **out, int device, const lora_target *targets, int n_targets, int r_max,
                     int n_slots, size_t page_bytes, void *pool_mem, size_t pool_bytes,
                     uint64_t scatter_seed) {
  if (!out) return LORA_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_shape(targets, n_targets, r_max, n_slots, page_bytes);
  if (rc != LORA_OK) return rc;
  if (!pool_mem) return LORA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(pool_mem) & 255u) return LORA_ERR_ALIGNMENT;
  int n_dev = 0;
  CUDA_TRY(cudaGetDeviceCount(&n_dev));
  if (device < 0 || device >= n_dev) return LORA_ERR_INVALID_ARG;

  lora_pool *p = new (std::nothrow) lora_pool();
  if (!p) return LORA_ERR_INVALID_ARG;
  p->device = device;
  p->n_targets = n_targets;
  p->r_max = r_max;
  p->n_slots = n_slots;
  p->targets.assign(targets, targets + n_targets);
  p->slot_bytes = slot_layout(targets, n_targets, r_max, &p->a_off, &p->bt_off);
  if (page_bytes == 0) {
    p->page_bytes = (long long)align256(size_t(p->slot_bytes));
    p->pps = 1;
    p->log2_page = -1;
  } else {
    p->page_bytes = (long long)page_bytes;
    p->pps = (int)((p->slot_bytes + p->page_bytes - 1) / p->page_bytes);
    int lg = 0;
    while ((1ll << lg) < p->page_bytes) ++lg;
    p->log2_page = (p->pps == 1) ? -1 : lg;
  }
  long long n_pages = (long long)(pool_bytes / (size_t)p->page_bytes);
  if (n_pages < 1 || n_pages > (1ll << 31) - 1) {
    delete p;
    return LORA_ERR_INVALID_ARG;
  }
  p->n_pages = (int)n_pages;
  p->mem = static_cast<uint8_t *>(pool_mem);
  p->mem_bytes = pool_bytes;

  // free list: ascending, or a seeded permutation; handed out from the front
  std::vector<int32_t> order(p->n_pages);
  for (int i = 0; i < p->n_pages; ++i) order[i] = i;
  if (scatter_seed != 0) {
    uint64_t s = scatter_seed;
    for (int i = p->n_pages - 1; i > 0; --i) {
      int j = (int)(splitmix64(s) % (uint64_t)(i + 1));
      std::swap(order[i], order[j]);
    }
  }
  p->free_pages.assign(order.rbegin(), order.rend());

  p->pt.assign((size_t)n_slots * p->pps, -1);
  p->rank.assign((size_t)n_slots * n_targets, 0);
  p->loaded.assign((size_t)n_slots, 0);

  DeviceGuard g(device);
  size_t pt_b = align256(p->pt.size() * 4), rk_b = align256(p->rank.size() * 4),
         ld_b = align256(p->loaded.size() * 4);
  if (cudaMalloc(&p->dev_tables, pt_b + rk_b + ld_b + 256) != cudaSuccess) {
    (void)cudaGetLastError();
    delete p;
    return LORA_ERR_CUDA;
  }
  uint8_t *b = static_cast<uint8_t *>(p->dev_tables);
  p->d_pt = reinterpret_cast<int32_t *>(b);
  p->d_rank = reinterpret_cast<int32_t *>(b + pt_b);
  p->d_loaded = reinterpret_cast<int32_t *>(b + pt_b + rk_b);
  p->d_status = reinterpret_cast<int *>(b + pt_b + rk_b + ld_b);
  bool ok = cudaMemcpy(p->d_pt, p->pt.data(), p->pt.size() * 4, cudaMemcpyHostToDevice) == cudaSuccess &&
            cudaMemset(p->d_rank, 0, p->rank.size() * 4) == cudaSuccess &&
            cudaMemset(p->d_loaded, 0, p->loaded.size() * 4) == cudaSuccess &&
            cudaMemset(p->d_status, 0, 4) == cudaSuccess && decode_setup(p) == LORA_OK;
  if (!ok) {
    (void)cudaGetLastError();
    cudaFree(p->dev_tables);
    delete p;
    return LORA_ERR_CUDA;
  }
  *out = p;
  return LORA_OK;
}

int lora_pool_load(lora_pool *p, int slot, int target, int rank, const void *A, const void *B,
                   int src_is_device, void *stream) {
  NvtxRange nvtx_range("lora_pool_load");
  if (!p) return LORA_ERR_INVALID_ARG;
  if (slot < 0 || slot >= p->n_slots) return LORA_ERR_SLOT;
  if (target < 0 || target >= p->n_targets) return LORA_ERR_INVALID_ARG;
  if (rank < 0 || rank > p->r_max) return LORA_ERR_INVALID_ARG;
  if (rank > 0 && (!A || !B)) return LORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(p->mu);
  DeviceGuard g(p->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int d_in = p->targets[target].d_in, d_out = p->targets[target].d_out;

  if (!p->loaded[slot]) {
    if ((int)p->free_pages.size() < p->pps) return LORA_ERR_NO_PAGES;
    for (int i = 0; i < p->pps; ++i) {
      p->pt[(size_t)slot * p->pps + i] = p->free_pages.back();
      p->free_pages.pop_back();
    }
    p->loaded[slot] = 1;
    CUDA_TRY(cudaMemcpyAsync(p->d_pt + (size_t)slot * p->pps, p->pt.data() + (size_t)slot * p->pps,
                             (size_t)p->pps * 4, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(p->d_loaded + slot, p->loaded.data() + slot, 4, cudaMemcpyHostToDevice, st));
  }

  const long long a_off = p->a_off[target], bt_off = p->bt_off[target];
  const long long a_all = (long long)p->r_max * d_in * 2, b_all = (long long)p->r_max * d_out * 2;
  int rc = LORA_OK;
  if (src_is_device) {
    // one kernel per block: the rows in the pool's tiled arrangement, B
    // transposed, the rank padding zeroed
    const int threads = 256;
    const long long na = (long long)p->r_max * (d_in / 8), nb = (long long)p->r_max * (d_out / 8);
    g_launches.fetch_add(2);
    store_block_kernel<<<(unsigned)((na + threads - 1) / threads), threads, 0, st>>>(
        p->view(), slot, a_off, d_in, p->r_max, rank, static_cast<const uint16_t *>(A), 0);
    store_block_kernel<<<(unsigned)((nb + threads - 1) / threads), threads, 0, st>>>(
        p->view(), slot, bt_off, d_out, p->r_max, rank, static_cast<const uint16_t *>(B), 1);
    if (cudaGetLastError() != cudaSuccess) rc = LORA_ERR_CUDA;
  } else {
    // host images of both blocks, each copied as one logical range (cut at
    // page boundaries)
    std::vector<uint16_t> ia, ib;
    block_image(static_cast<const uint16_t *>(A), 0, d_in, p->r_max, rank, &ia);
    block_image(static_cast<const uint16_t *>(B), 1, d_out, p->r_max, rank, &ib);
    auto copy = [&](const uint8_t *src) {
      return [&, src](uint8_t *dst, long long done, long long n) {
        if (rc == LORA_OK && cudaMemcpyAsync(dst, src + done, (size_t)n, cudaMemcpyHostToDevice, st) != cudaSuccess)
          rc = LORA_ERR_CUDA;
      };
    };
    for_each_run(p, slot, a_off, a_all, copy(reinterpret_cast<const uint8_t *>(ia.data())));
    for_each_run(p, slot, bt_off, b_all, copy(reinterpret_cast<const uint8_t *>(ib.data())));
    if (rc == LORA_OK && cudaStreamSynchronize(st) != cudaSuccess) rc = LORA_ERR_CUDA;  // the images go out of scope
  }
  if (rc != LORA_OK) {
    (void)cudaGetLastError();
    return rc;
  }
  p->rank[(size_t)slot * p->n_targets + target] = rank;
  CUDA_TRY(cudaMemcpyAsync(p->d_rank + (size_t)slot * p->n_targets + target,
                           p->rank.data() + (size_t)slot * p->n_targets + target, 4,
                           cudaMemcpyHostToDevice, st));
  return LORA_OK;
}

size_t lora_swap_src_bytes(const lora_pool *p, const int *ranks) {
  if (!p || !ranks) return 0;
  const long long n = swap_src_bytes(p, ranks);
  return n < 0 ? 0 : size_t(n);
}

size_t lora_swap_staging_bytes(const lora_pool *p, const int *ranks) {
  if (!p || !ranks) return 0;
  const long long n = swap_src_bytes(p, ranks);
  return n < 0 ? 0 : swap_desc_bytes(p) + size_t(n);
}

int lora_pool_swap_in(lora_pool *p, int slot, const int *ranks, const void *src, size_t src_bytes, void *staging,
                      size_t staging_bytes, void *stream) {
  NvtxRange nvtx_range("lora_pool_swap_in");
  if (!p || !ranks) return LORA_ERR_INVALID_ARG;
  if (slot < 0 || slot >= p->n_slots) return LORA_ERR_SLOT;
  const long long need = swap_src_bytes(p, ranks);
  if (need < 0 || (long long)src_bytes != need) return LORA_ERR_INVALID_ARG;
  if (need > 0 && !src) return LORA_ERR_INVALID_ARG;
  if (!staging) return LORA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(staging) & 255u) return LORA_ERR_ALIGNMENT;
  if (staging_bytes < swap_desc_bytes(p) + size_t(need)) return LORA_ERR_WORKSPACE;
  std::lock_guard<std::mutex> lk(p->mu);
  DeviceGuard g(p->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!p->loaded[slot]) {
    if ((int)p->free_pages.size() < p->pps) return LORA_ERR_NO_PAGES;
    for (int i = 0; i < p->pps; ++i) {
      p->pt[(size_t)slot * p->pps + i] = p->free_pages.back();
      p->free_pages.pop_back();
    }
    p->loaded[slot] = 1;
    CUDA_TRY(cudaMemcpyAsync(p->d_pt + (size_t)slot * p->pps, p->pt.data() + (size_t)slot * p->pps,
                             (size_t)p->pps * 4, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(p->d_loaded + slot, p->loaded.data() + slot, 4, cudaMemcpyHostToDevice, st));
  }
  // descriptors (a small pageable copy, staged by the driver before the call
  // returns), then the adapter itself in one copy, then one scatter kernel
  std::vector<SwapDesc> desc(p->n_targets);
  long long off = 0, widest = 0;
  for (int t = 0; t < p->n_targets; ++t) {
    SwapDesc &d = desc[t];
    d.src = off;
    d.a_off = p->a_off[t];
    d.bt_off = p->bt_off[t];
    d.pad = 0;
    d.d_in = p->targets[t].d_in;
    d.d_out = p->targets[t].d_out;
    d.rank = ranks[t];
    d.pad2 = 0;
    off += (long long)ranks[t] * (d.d_in + d.d_out) * 2;
    widest = std::max(widest, (long long)p->r_max * (d.d_in + d.d_out) / 8);
  }
  uint8_t *stg = static_cast<uint8_t *>(staging);
  CUDA_TRY(cudaMemcpyAsync(stg, desc.data(), desc.size() * sizeof(SwapDesc), cudaMemcpyHostToDevice, st));
  if (need > 0) CUDA_TRY(cudaMemcpyAsync(stg + swap_desc_bytes(p), src, (size_t)need, cudaMemcpyHostToDevice, st));
  const int threads = 256;
  const unsigned bx = (unsigned)std::min<long long>(64, (widest + threads - 1) / threads);
  g_launches.fetch_add(1);
  swap_in_kernel<<<dim3(bx, (unsigned)p->n_targets), threads, 0, st>>>(
      p->view(), slot, p->r_max, reinterpret_cast<const SwapDesc *>(stg), stg + swap_desc_bytes(p));
  CUDA_TRY(cudaGetLastError());
  for (int t = 0; t < p->n_targets; ++t) p->rank[(size_t)slot * p->n_targets + t] = ranks[t];
  CUDA_TRY(cudaMemcpyAsync(p->d_rank + (size_t)slot * p->n_targets, p->rank.data() + (size_t)slot * p->n_targets,
                           (size_t)p->n_targets * 4, cudaMemcpyHostToDevice, st));
  return LORA_OK;
}

int lora_pool_unload(lora_pool *p, int slot) {
  if (!p) return LORA_ERR_INVALID_ARG;
  if (slot < 0 || slot >= p->n_slots) return LORA_ERR_SLOT;
  std::lock_guard<std::mutex> lk(p->mu);
  if (!p->loaded[slot]) return LORA_ERR_NOT_LOADED;
  DeviceGuard g(p->device);
  CUDA_TRY(cudaDeviceSynchronize());
  for (int i = p->pps - 1; i >= 0; --i) {
    p->free_pages.push_back(p->pt[(size_t)slot * p->pps + i]);
    p->pt[(size_t)slot * p->pps + i] = -1;
  }
  for (int t = 0; t < p->n_targets; ++t) p->rank[(size_t)slot * p->n_targets + t] = 0;
  p->loaded[slot] = 0;
  CUDA_TRY(cudaMemcpy(p->d_pt + (size_t)slot * p->pps, p->pt.data() + (size_t)slot * p->pps,
                      (size_t)p->pps * 4, cudaMemcpyHostToDevice));
  CUDA_TRY(cudaMemcpy(p->d_rank + (size_t)slot * p->n_targets, p->rank.data() + (size_t)slot * p->n_targets,
                      (size_t)p->n_targets * 4, cudaMemcpyHostToDevice));
  CUDA_TRY(cudaMemcpy(p->d_loaded + slot, p->loaded.data() + slot, 4, cudaMemcpyHostToDevice));
  return LORA_OK;
}

int lora_pool_destroy(lora_pool *p) {
  if (!p) return LORA_ERR_INVALID_ARG;
  int rc = LORA_OK;
  {
    DeviceGuard g(p->device);
    if (cudaDeviceSynchronize() != cudaSuccess) rc = LORA_ERR_CUDA;
    if (p->dev_tables && cudaFree(p->dev_tables) != cudaSuccess) rc = LORA_ERR_CUDA;
    (void)cudaGetLastError();
  }
  delete p;
  return rc;
}

const int32_t *lora_pool_page_table(const lora_pool *p) { return p ? p->d_pt : nullptr; }

int lora_pool_get_info(const lora_pool *p, lora_pool_info *info) {
  if (!p || !info) return LORA_ERR_INVALID_ARG;
  info->slot_bytes = (size_t)p->slot_bytes;
  info->page_bytes = (size_t)p->page_bytes;
  info->pages_per_slot = p->pps;
  info->n_pages = p->n_pages;
  info->free_pages = (int)p->free_pages.size();
  info->n_slots = p->n_slots;
  info->n_targets = p->n_targets;
  info->r_max = p->r_max;
  info->decode_ctas = p->decode_max_ctas;
  return LORA_OK;
}

int lora_pool_target_offsets(const lora_pool *p, int target, size_t *a_off, size_t *bt_off) {
  if (!p || target < 0 || target >= p->n_targets || !a_off || !bt_off) return LORA_ERR_INVALID_ARG;
  *a_off = (size_t)p->a_off[target];
  *bt_off = (size_t)p->bt_off[target];
  return LORA_OK;
}

uint64_t lora_kernel_launches(void) { return g_launches.load(); }

int lora_get_error(lora_pool *p, int *device_status, void *stream) {
  if (!p || !device_status) return LORA_ERR_INVALID_ARG;
  DeviceGuard g(p->device);
  CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int v = 0;
  CUDA_TRY(cudaMemcpy(&v, p->d_status, 4, cudaMemcpyDeviceToHost));
  CUDA_TRY(cudaMemset(p->d_status, 0, 4));
  *device_status = v;
  return LORA_OK;
}

}  // extern "C"
