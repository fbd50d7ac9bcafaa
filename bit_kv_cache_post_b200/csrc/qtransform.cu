// Query transform q' = T_k^{-T} q (summary page "WUSH-KV：数据自适应变换的 KV
// Cache 低比特量化", 方法关键点 and 工作参考价值: one d x d product per query;
// the inverse transpose keeps q'.k' = q.k).  One CTA per (sequence, KV head)
// transforms the G query heads of that group: thread i streams row i of the
// group's matrix (staged in shared memory with coalesced loads; L2-resident
// across the batch) against the G query vectors.
#include "wushkv_internal.cuh"

namespace wushkv {

namespace {

template <int G>
__global__ void __launch_bounds__(128) qtransform_kernel(const void* q, int dtype,
                                                         const float* TinvT, float* out,
                                                         int n_kv_heads) {
  extern __shared__ __align__(16) float qsm[];
  query_transform_unit<G>(q, dtype, TinvT, out, blockIdx.x / n_kv_heads, blockIdx.x % n_kv_heads,
                          n_kv_heads, qsm);
}

}  // namespace

cudaError_t launch_query_transform(const void* q, int dtype, const float* TinvT, float* out,
                                   int batch, int n_q_heads, int n_kv_heads, cudaStream_t s) {
  const int G = n_q_heads / n_kv_heads;
  const unsigned grid = (unsigned)(batch * n_kv_heads);
  const size_t smem = query_transform_smem(G);
  auto go = [&](auto kern) -> cudaError_t {
    int dev = 0;
    cudaGetDevice(&dev);
    static int done[64][5] = {};
    const int gi = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : 4;
    if (dev < 64 && !done[dev][gi]) {
      const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      done[dev][gi] = 1;
    }
    kern<<<grid, 128, smem, s>>>(q, dtype, TinvT, out, n_kv_heads);
    return cudaSuccess;
  };
  cudaError_t e;
  switch (G) {
    case 1: e = go(qtransform_kernel<1>); break;
    case 2: e = go(qtransform_kernel<2>); break;
    case 4: e = go(qtransform_kernel<4>); break;
    case 8: e = go(qtransform_kernel<8>); break;
    case 16: e = go(qtransform_kernel<16>); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace wushkv
