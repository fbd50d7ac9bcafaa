// Query transform q' = T_k^{-T} q (summary page "WUSH-KV：数据自适应变换的 KV
// Cache 低比特量化", 方法关键点 and 工作参考价值: one d x d product per query;
// the inverse transpose keeps q'.k' = q.k).  One CTA per (sequence, KV head)
// transforms the G query heads of that group with one staged copy of the
// group's matrix.
#include "wushkv_internal.cuh"

namespace wushkv {

namespace {

constexpr int MT_LD = 129;

__device__ __forceinline__ float load_q(const void* p, int dtype, size_t i) {
  if (dtype == WUSHKV_F16) return __half2float(static_cast<const __half*>(p)[i]);
  if (dtype == WUSHKV_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
  return static_cast<const float*>(p)[i];
}

__global__ void __launch_bounds__(128) qtransform_kernel(const void* q, int dtype,
                                                         const float* TinvT, float* out,
                                                         int n_q_heads, int n_kv_heads) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Mt = reinterpret_cast<float*>(smem_raw);  // [128][MT_LD] = M^T
  float* qs = Mt + D * MT_LD;                      // [G][128]
  const int G = n_q_heads / n_kv_heads;
  const int b = blockIdx.x / n_kv_heads, h = blockIdx.x % n_kv_heads;
  const int tid = threadIdx.x;
  stage_transpose_128(TinvT + (size_t)h * D * D, Mt, MT_LD);
  for (int g = 0; g < G; ++g)
    qs[g * D + tid] = load_q(q, dtype, ((size_t)b * n_q_heads + (size_t)h * G + g) * D + tid);
  __syncthreads();
  for (int g = 0; g < G; ++g) {
    const float* qg = qs + g * D;
    float acc = 0.f;
#pragma unroll 8
    for (int j = 0; j < D; ++j) acc = fmaf(Mt[j * MT_LD + tid], qg[j], acc);
    out[((size_t)b * n_q_heads + (size_t)h * G + g) * D + tid] = acc;
  }
}

}  // namespace

cudaError_t launch_query_transform(const void* q, int dtype, const float* TinvT, float* out,
                                   int batch, int n_q_heads, int n_kv_heads, cudaStream_t s) {
  const int G = n_q_heads / n_kv_heads;
  const size_t smem = (size_t)(D * MT_LD + G * D) * sizeof(float);
  int dev = 0;
  cudaGetDevice(&dev);
  static int attr_done[64] = {0};
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(qtransform_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(D * MT_LD * sizeof(float) + 16 * D * sizeof(float)));
    if (e != cudaSuccess) return e;
    attr_done[dev] = 1;
  }
  qtransform_kernel<<<batch * n_kv_heads, 128, smem, s>>>(q, dtype, TinvT, out, n_q_heads,
                                                           n_kv_heads);
  return cudaGetLastError();
}

}  // namespace wushkv
