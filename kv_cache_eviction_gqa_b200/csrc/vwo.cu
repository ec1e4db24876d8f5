// ||V_i W_O^h||_1 for every row i and query head h of a kv-head group
// ("Resumo Técnico: CriticalKV", Framework Teórico: the perturbation bound depends on the
// projected values V W_O; Algoritmo, Etapa 2: A_i * ||V_i W_O||_1).
//
// out[g][r][j] = sum_c | sum_d V[g][r][d] * W_O[(kvh*G + j)*D + d][c] |, kvh = g % Hkv.
// This file holds the dispatcher and a CUDA-core kernel for widths the tensor-core kernel
// (vwo_tc.cu) does not tile (hidden not a multiple of 128).
#include "qe_internal.cuh"

namespace {

// CUDA-core reference kernel: 64 rows x 64 columns per tile, K = D in one shot.
// Used for shapes the tensor-core kernel does not take.
template <typename T, int D>
__global__ void __launch_bounds__(256) vwo_simt_kernel(const T* V, int rows, const T* W, int Hkv,
                                                       int G, int hidden, float* out, long long ogs) {
  __shared__ float Vs[64][D + 1];
  __shared__ float Ws[32][64 + 4];
  const int g = blockIdx.y / G, j = blockIdx.y % G, kvh = g % Hkv;
  const int r0 = blockIdx.x * 64;
  const int tid = threadIdx.x, tr = tid / 16, tc = tid % 16;
  const T* Vg = V + (size_t)g * rows * D;
  const T* Wh = W + (size_t)(kvh * G + j) * D * hidden;
  for (int i = tid; i < 64 * D; i += 256) {
    const int r = i / D, d = i % D;
    Vs[r][d] = (r0 + r < rows) ? Elem<T>::to_f(Vg[(size_t)(r0 + r) * D + d]) : 0.f;
  }
  float rs[4] = {0.f, 0.f, 0.f, 0.f};
  for (int c0 = 0; c0 < hidden; c0 += 64) {
    float acc[4][4] = {};
    for (int d0 = 0; d0 < D; d0 += 32) {
      __syncthreads();
      for (int i = tid; i < 32 * 64; i += 256) {
        const int d = i / 64, c = i % 64;
        Ws[d][c] = Elem<T>::to_f(Wh[(size_t)(d0 + d) * hidden + c0 + c]);
      }
      __syncthreads();
      for (int d = 0; d < 32; ++d) {
        float a[4], bb[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) a[x] = Vs[tr * 4 + x][d0 + d];
#pragma unroll
        for (int y = 0; y < 4; ++y) bb[y] = Ws[d][tc * 4 + y];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(a[x], bb[y], acc[x][y]);
      }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) rs[x] += fabsf(acc[x][y]);
  }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    float v = rs[x];
#pragma unroll
    for (int o = 8; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int r = r0 + tr * 4 + x;
    if (tc == 0 && r < rows) out[(size_t)g * ogs + (size_t)r * G + j] = v;
  }
}

template <typename T, int D>
int launch_simt(const void* V, int n_groups, int rows, const void* W, int Hq, int Hkv, int hidden,
                float* out, long long ogs, cudaStream_t s) {
  const int G = Hq / Hkv;
  dim3 grid((rows + 63) / 64, n_groups * G);
  vwo_simt_kernel<T, D><<<grid, 256, 0, s>>>((const T*)V, rows, (const T*)W, Hkv, G, hidden, out, ogs);
  return cudaGetLastError() == cudaSuccess ? QE_OK : QE_ERR_CUDA;
}

}  // namespace

int launch_vwo_simt(const void* V, int n_groups, int rows, int D, int dtype, const void* W_O, int Hq,
                    int Hkv, int hidden, float* out, long long ogs, cudaStream_t s) {
  const bool bf = dtype == QE_BF16;
  if (D == 128)
    return bf ? launch_simt<__nv_bfloat16, 128>(V, n_groups, rows, W_O, Hq, Hkv, hidden, out, ogs, s)
              : launch_simt<__half, 128>(V, n_groups, rows, W_O, Hq, Hkv, hidden, out, ogs, s);
  return bf ? launch_simt<__nv_bfloat16, 64>(V, n_groups, rows, W_O, Hq, Hkv, hidden, out, ogs, s)
            : launch_simt<__half, 64>(V, n_groups, rows, W_O, Hq, Hkv, hidden, out, ogs, s);
}

int launch_vwo(const void* V, int n_groups, int rows, int D, int dtype, const void* W_O, int Hq,
               int Hkv, int hidden, float* out, long long ogs, int32_t* status, cudaStream_t s) {
  if (hidden % 128 == 0)
    return launch_vwo_tc(V, n_groups, rows, D, dtype, W_O, Hq, Hkv, hidden, out, ogs, status, s);
  return launch_vwo_simt(V, n_groups, rows, D, dtype, W_O, Hq, Hkv, hidden, out, ogs, s);
}
