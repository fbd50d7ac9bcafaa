// Query transform q' = T_k^{-T} q (summary page "WUSH-KV：数据自适应变换的 KV
// Cache 低比特量化", 方法关键点 and 工作参考价值: one d x d product per query;
// the inverse transpose keeps q'.k' = q.k).  One CTA per (sequence, KV head)
// transforms the G query heads of that group: thread i streams row i of the
// group's matrix (each warp 32 rows, eight coalesced 512-byte row loads at a
// time; L2-resident across the batch) against the G query vectors.
#include "wushkv_internal.cuh"

namespace wushkv {

namespace {

template <int G>
__global__ void __launch_bounds__(128) qtransform_kernel(const void* q, int dtype,
                                                         const float* TinvT, float* out,
                                                         int n_kv_heads) {
  query_transform_unit<G>(q, dtype, TinvT, out, blockIdx.x / n_kv_heads, blockIdx.x % n_kv_heads,
                          n_kv_heads);
}

}  // namespace

cudaError_t launch_query_transform(const void* q, int dtype, const float* TinvT, float* out,
                                   int batch, int n_q_heads, int n_kv_heads, cudaStream_t s) {
  const int G = n_q_heads / n_kv_heads;
  const unsigned grid = (unsigned)(batch * n_kv_heads);
  switch (G) {
    case 1: qtransform_kernel<1><<<grid, 128, 0, s>>>(q, dtype, TinvT, out, n_kv_heads); break;
    case 2: qtransform_kernel<2><<<grid, 128, 0, s>>>(q, dtype, TinvT, out, n_kv_heads); break;
    case 4: qtransform_kernel<4><<<grid, 128, 0, s>>>(q, dtype, TinvT, out, n_kv_heads); break;
    case 8: qtransform_kernel<8><<<grid, 128, 0, s>>>(q, dtype, TinvT, out, n_kv_heads); break;
    case 16: qtransform_kernel<16><<<grid, 128, 0, s>>>(q, dtype, TinvT, out, n_kv_heads); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace wushkv
