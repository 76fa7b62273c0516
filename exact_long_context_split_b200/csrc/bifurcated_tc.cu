// The bifurcated tensor-core kernels and their launchers.
#include "bifurcated_tc.cuh"

namespace ta {

size_t bif_prefix_smem_bytes() { return sizeof(BifSmem) + 1024; }

cudaError_t bif_prefix_set_smem_limit() {
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(&bif_prefix_kernel<false>),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bif_prefix_smem_bytes()));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(reinterpret_cast<const void*>(&bif_prefix_kernel<true>),
                              cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bif_prefix_smem_bytes()));
}

cudaError_t launch_bif_prefix(dim3 grid, const CUtensorMap& kmap, const CUtensorMap& vmap, const BifParams& p,
                              cudaStream_t st) {
  if (p.mode == 1 && p.block_table != nullptr)
    bif_prefix_kernel<true><<<grid, kBifThreads, bif_prefix_smem_bytes(), st>>>(kmap, vmap, p);
  else
    bif_prefix_kernel<false><<<grid, kBifThreads, bif_prefix_smem_bytes(), st>>>(kmap, vmap, p);
  return cudaGetLastError();
}

cudaError_t launch_merge_chunks(const float* part, int n_chunks, int n_kv_heads, int rows_per_head, int n_queries,
                                float* out, float* lse, int batch, int n_q_heads, const int* err, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(batch) * n_queries * n_q_heads * (kBifD / 4);  // one thread per 4 columns
  if (n == 0) return cudaSuccess;
  // Launched as a dependent of the tensor-core pass before it (programmatic dependent launch):
  // its blocks are scheduled while that kernel's last CTAs run and wait for its completion.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((n + 127) / 128));
  cfg.blockDim = dim3(128);
  cfg.stream = st;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = la;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_chunks_kernel, part, n_chunks, n_kv_heads, rows_per_head, n_queries, out,
                            lse, batch, n_q_heads, err);
}

}  // namespace ta
