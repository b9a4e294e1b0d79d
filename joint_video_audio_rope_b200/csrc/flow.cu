// Flow-matching elementwise kernels (digest step 4): the noised input
// z_t = t z_0 + (1 - t) eps with the velocity target u = z_0 - eps in one
// pass, and the per-item loss term ||v - (z_0 - eps)||^2.  Both are HBM-bound
// streams: 16-byte vector loads and stores, a grid of a few blocks per SM per
// batch item, the ragged end of each item (n not a multiple of the vector
// width) done by block 0 with scalar accesses.  The loss sums in fp32 in a
// fixed order (per-thread strided sums, a block tree, then one warp per item
// over the blocks' partials), so a call gives the same bits every time.
#include "internal.h"

namespace mmdit {

namespace {

template <typename T>
struct Vec;  // 16 bytes of T as fp32 values
template <>
struct Vec<float> {
  static constexpr int kN = 4;
  __device__ __forceinline__ static void load(const float* p, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  __device__ __forceinline__ static void store(float* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
  __device__ __forceinline__ static float get(const float* p) { return *p; }
  __device__ __forceinline__ static void put(float* p, float x) { *p = x; }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __float22bfloat162_rn(make_float2(x[2 * i], x[2 * i + 1]));
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __device__ __forceinline__ static float get(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ __forceinline__ static void put(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

constexpr int kThreads = 256;
constexpr int kTargetBlocks = 148 * 8;  // resident blocks of 256 threads on the B200

// Blocks per batch item: enough vectors per thread to keep loads in flight,
// the whole grid about one wave.
int blocks_per_item(int batch, long long n_vec) {
  const long long need = (n_vec + kThreads - 1) / kThreads;
  const long long cap = std::max(1, kTargetBlocks / std::max(1, batch));
  return (int)std::max(1LL, std::min(need, cap));
}

template <typename T>
__global__ void __launch_bounds__(kThreads) flow_noise_kernel(const T* __restrict__ z0,
                                                              const T* __restrict__ eps,
                                                              const float* __restrict__ t,
                                                              T* __restrict__ zt, T* __restrict__ u,
                                                              long long n, long long stride) {
  constexpr int V = Vec<T>::kN;
  const int b = blockIdx.y;
  const float tb = t[b];
  const long long base = (long long)b * stride;
  const long long n_vec = n / V;
  for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < n_vec;
       i += (long long)gridDim.x * kThreads) {
    float a[V], e[V], r[V];
    Vec<T>::load(z0 + base + i * V, a);
    Vec<T>::load(eps + base + i * V, e);
    if (zt != nullptr) {
#pragma unroll
      for (int j = 0; j < V; ++j) r[j] = tb * a[j] + (1.f - tb) * e[j];
      Vec<T>::store(zt + base + i * V, r);
    }
    if (u != nullptr) {
#pragma unroll
      for (int j = 0; j < V; ++j) r[j] = a[j] - e[j];
      Vec<T>::store(u + base + i * V, r);
    }
  }
  if (blockIdx.x == 0 && threadIdx.x < n - n_vec * V) {  // ragged end of the item
    const long long i = base + n_vec * V + threadIdx.x;
    const float a = Vec<T>::get(z0 + i), e = Vec<T>::get(eps + i);
    if (zt != nullptr) Vec<T>::put(zt + i, tb * a + (1.f - tb) * e);
    if (u != nullptr) Vec<T>::put(u + i, a - e);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) flow_loss_kernel(const T* __restrict__ v,
                                                             const T* __restrict__ z0,
                                                             const T* __restrict__ eps,
                                                             float* __restrict__ partial,
                                                             long long n, long long stride) {
  constexpr int V = Vec<T>::kN;
  const int b = blockIdx.y;
  const long long base = (long long)b * stride;
  const long long n_vec = n / V;
  float acc = 0.f;
  for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < n_vec;
       i += (long long)gridDim.x * kThreads) {
    float x[V], a[V], e[V];
    Vec<T>::load(v + base + i * V, x);
    Vec<T>::load(z0 + base + i * V, a);
    Vec<T>::load(eps + base + i * V, e);
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const float d = x[j] - (a[j] - e[j]);
      acc = fmaf(d, d, acc);
    }
  }
  if (blockIdx.x == 0 && threadIdx.x < n - n_vec * V) {
    const long long i = base + n_vec * V + threadIdx.x;
    const float d = Vec<T>::get(v + i) - (Vec<T>::get(z0 + i) - Vec<T>::get(eps + i));
    acc = fmaf(d, d, acc);
  }
  // block tree: warp shuffles, then the eight warp sums
  __shared__ float warp_sum[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float s = threadIdx.x < kThreads / 32 ? warp_sum[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) partial[(long long)b * gridDim.x + blockIdx.x] = s;
  }
}

// loss[b] = sum of the item's block partials; one warp per item.
__global__ void __launch_bounds__(32) flow_loss_final_kernel(const float* __restrict__ partial,
                                                             int blocks, float* __restrict__ loss) {
  const int b = blockIdx.x;
  float s = 0.f;
  for (int i = threadIdx.x; i < blocks; i += 32) s += partial[(long long)b * blocks + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (threadIdx.x == 0) loss[b] = s;
}

int check_flow(const char* who, int batch, long long n, long long stride, int dtype,
               std::initializer_list<const void*> ptrs) {
  if (batch < 1 || batch > 65535 || n < 0 || stride < n)  // batch items are grid rows
    return fail(MMDIT_EINVAL, "%s: batch %d, n %lld, stride %lld out of range", who, batch, n, stride);
  if (dtype != MMDIT_BF16 && dtype != MMDIT_F32)
    return fail(MMDIT_EUNSUPPORTED, "%s: dtype %d not supported", who, dtype);
  const int es = dtype == MMDIT_BF16 ? 2 : 4;
  if ((stride * es) % 16 != 0)
    return fail(MMDIT_EINVAL, "%s: stride * element size must be a multiple of 16 bytes", who);
  for (const void* p : ptrs)
    if (p != nullptr && !aligned16(p))
      return fail(MMDIT_EINVAL, "%s: tensors must be 16-byte aligned", who);
  return MMDIT_OK;
}

}  // namespace

}  // namespace mmdit

using namespace mmdit;

extern "C" {

int mmdit_flow_noise(const void* z0, const void* eps, const float* t, void* zt, void* u,
                     int32_t batch, int64_t n, int64_t stride, int32_t dtype,
                     mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_flow_noise");
  int rc = check_flow("flow_noise", batch, n, stride, dtype, {z0, eps, zt, u});  // t: scalar reads
  if (rc) return rc;
  if (!z0 || !eps || !t) return fail(MMDIT_EINVAL, "flow_noise: z0, eps, t must be non-NULL");
  if (!zt && !u) return fail(MMDIT_EINVAL, "flow_noise: zt and u are both NULL");
  if (n == 0) return MMDIT_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == MMDIT_BF16) {
    const dim3 grid(blocks_per_item(batch, n / 8), batch);
    flow_noise_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
        (const __nv_bfloat16*)z0, (const __nv_bfloat16*)eps, t, (__nv_bfloat16*)zt,
        (__nv_bfloat16*)u, n, stride);
  } else {
    const dim3 grid(blocks_per_item(batch, n / 4), batch);
    flow_noise_kernel<float><<<grid, kThreads, 0, s>>>((const float*)z0, (const float*)eps, t,
                                                       (float*)zt, (float*)u, n, stride);
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "flow_noise launch");
}

size_t mmdit_flow_loss_workspace_size(int32_t batch, int64_t n) {
  if (batch < 1 || n < 0) return 0;
  // the fp32 vector count bounds the bf16 one, so this covers both dtypes
  return align256((size_t)batch * blocks_per_item(batch, n / 4) * sizeof(float));
}

int mmdit_flow_loss(const void* v, const void* z0, const void* eps, float* loss, int32_t batch,
                    int64_t n, int64_t stride, int32_t dtype, void* workspace, size_t ws_bytes,
                    mmdit_stream_t stream) {
  MMDIT_NVTX("mmdit_flow_loss");
  int rc = check_flow("flow_loss", batch, n, stride, dtype, {v, z0, eps});
  if (rc) return rc;
  if (!v || !z0 || !eps || !loss)
    return fail(MMDIT_EINVAL, "flow_loss: v, z0, eps, loss must be non-NULL");
  const size_t need = mmdit_flow_loss_workspace_size(batch, n);
  if (workspace == nullptr || ws_bytes < need)
    return fail(MMDIT_EWORKSPACE, "flow_loss: workspace needs %zu bytes", need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(MMDIT_EINVAL, "flow_loss: workspace must be 256-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  float* partial = static_cast<float*>(workspace);
  int blocks;
  if (dtype == MMDIT_BF16) {
    blocks = blocks_per_item(batch, n / 8);
    flow_loss_kernel<__nv_bfloat16><<<dim3(blocks, batch), kThreads, 0, s>>>(
        (const __nv_bfloat16*)v, (const __nv_bfloat16*)z0, (const __nv_bfloat16*)eps, partial, n,
        stride);
  } else {
    blocks = blocks_per_item(batch, n / 4);
    flow_loss_kernel<float><<<dim3(blocks, batch), kThreads, 0, s>>>(
        (const float*)v, (const float*)z0, (const float*)eps, partial, n, stride);
  }
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    flow_loss_final_kernel<<<batch, 32, 0, s>>>(partial, blocks, loss);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? MMDIT_OK : cuda_fail(e, "flow_loss launch");
}

}  // extern "C"
