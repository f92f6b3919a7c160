// Intermediate arrays of a score call, copied out of the engine's workspace
// for direct checks against their definitions: rho_j = 1/||k_j|| (GEMM form;
// stored per unit at 256-aligned offsets with zero pads) and U = sum_j k_j /
// ||k_j|| per unit (closed form; one partial sum per score chunk in the chunk
// statistics, added here in chunk order).
#include "rkv_internal.cuh"

namespace rkv {
namespace {

__global__ void gather_rho_kernel(const int64_t* __restrict__ tok_off,
                                  const int64_t* __restrict__ rho_off,
                                  const float* __restrict__ rho, float* __restrict__ out) {
  const int u = blockIdx.x;
  const int64_t t0 = tok_off[u];
  const int n = static_cast<int>(tok_off[u + 1] - t0);
  const float* src = rho + rho_off[u];
  for (int j = threadIdx.x; j < n; j += blockDim.x) out[t0 + j] = src[j];
}

__global__ void sum_unit_U_kernel(const int* __restrict__ chunk_off,
                                  const float* __restrict__ xstat, int xs, int u0,
                                  float* __restrict__ out) {
  const int u = blockIdx.x;
  const int d = threadIdx.x;   // 0 .. 127
  float acc = 0.f;
  for (int g = chunk_off[u]; g < chunk_off[u + 1]; ++g)
    acc += xstat[static_cast<int64_t>(g) * xs + u0 + d];
  out[static_cast<int64_t>(u) * kHeadDim + d] = acc;
}

}  // namespace

cudaError_t launch_gather_rho(const int64_t* tok_off, const int64_t* rho_off, int U,
                              const float* rho, float* out, cudaStream_t st) {
  gather_rho_kernel<<<U, 256, 0, st>>>(tok_off, rho_off, rho, out);
  return cudaGetLastError();
}

cudaError_t launch_sum_unit_U(const int* chunk_off, int U, const float* xstat, int xs, int u0,
                              float* out, cudaStream_t st) {
  sum_unit_U_kernel<<<U, kHeadDim, 0, st>>>(chunk_off, xstat, xs, u0, out);
  return cudaGetLastError();
}

}  // namespace rkv
