// moe.cu -- slots of routed expert pairs for batches too large to group in
// the delta kernel.
//
// In a mixture-of-experts layer each token is routed to top_k experts, and an
// adapted expert projection carries the adapter's own shrink and expand for
// that expert ("Multi-LoRA Serving: Sharing One GPU Across Adapters", section
// "MoE Models Raise the Bar").  The delta then runs over (token, expert)
// pairs, pair p = t * top_k + j: its slot in the pool is
// adapter(t) * n_experts + topk[p], its input the token's x row, its output
// the pair's own row of the expert output.  Up to 256 pairs the decode kernel
// forms the slots itself while it groups the rows; beyond that this kernel
// writes them for the plan kernel.
#include "internal.cuh"

namespace lora {

__global__ void moe_pair_ids_kernel(const int32_t *lora_ids, const int32_t *topk, int n_pairs, int top_k,
                                    int n_experts, int n_slots, int32_t *pair_ids) {
  griddep_wait();
  griddep_launch_dependents();
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < n_pairs; p += gridDim.x * blockDim.x) {
    const int lo = lora_ids[p / top_k];
    int s = -1;
    if (lo != -1) {
      const int e = topk[p];
      const long long v = (long long)lo * n_experts + e;
      s = (lo < -1 || e < 0 || e >= n_experts || v >= n_slots) ? n_slots : (int)v;  // n_slots: a bad id
    }
    pair_ids[p] = s;
  }
}

int launch_moe_pair_ids(const lora_pool *pool, const int32_t *lora_ids, const int32_t *topk, int n_pairs,
                        int top_k, int n_experts, int32_t *pair_ids, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((n_pairs + 255) / 256);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      cudaLaunchKernelEx(&cfg, moe_pair_ids_kernel, lora_ids, topk, n_pairs, top_k, n_experts, pool->n_slots, pair_ids);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  g_launches.fetch_add(1);
  return LORA_OK;
}

}  // namespace lora
