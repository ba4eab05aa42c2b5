// Grouped expert GEMM on the CUDA cores (FFMA, fp32 accumulate).
//
// The fp32 workload needs a 1e-5 relative bound, which tf32 tensor cores
// cannot meet, so fp32 inputs run here in true fp32.  The same problems and
// epilogues as the tcgen05 kernel (bias + GELU for the first expert layer,
// bias times gate for the second), 64 x 64 output tiles, 4 x 4 per thread.
// It also accepts bf16 and fp16 inputs, which gives a second GPU implementation to
// cross-check the tensor-core path.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kSBM = 64, kSBN = 64, kSBK = 16;

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs a) {
  __shared__ float As[kSBK][kSBM + 4];
  __shared__ float Bs[kSBK][kSBN + 4];
  __shared__ int poff[33], cnt[32];
  __shared__ int bad;
  const GemmProblem& pr = a.p[blockIdx.z];
  const int tid = threadIdx.x;
  if (tid == 0) {
    int p = 0;
    bad = 0;
    poff[0] = 0;
    if (pr.routed) {
      for (int e = 0; e < a.E; ++e) {
        int c = a.offsets[e + 1] - a.offsets[e];
        if (c < 0) { c = 0; bad = 1; }
        cnt[e] = c;
        p += (c + kSegAlign - 1) / kSegAlign * kSegAlign;
        poff[e + 1] = p;
      }
      if ((long long)p > a.r_max) bad = 1;
    }
  }
  __syncthreads();
  if (bad) {
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) set_status(a.status, DEV_BAD_INDEX, 400);
    return;
  }
  const int row0 = blockIdx.y * kSBM;
  const int n0 = blockIdx.x * kSBN;
  if (n0 >= pr.N) return;
  int e = 0, valid;
  if (pr.routed) {
    if (row0 >= poff[a.E]) return;
    while (e < a.E - 1 && row0 >= poff[e + 1]) ++e;
    valid = poff[e] + cnt[e] - row0;
  } else {
    valid = pr.M - row0;
  }
  if (valid <= 0) return;
  if (valid > kSBM) valid = kSBM;
  const T* A = reinterpret_cast<const T*>(pr.A) + (long long)row0 * pr.K;
  // B row n of expert e, element k; a K-split B is a stack [K/ksplit][N][ksplit]
  const T* Bbase = reinterpret_cast<const T*>(pr.B);
  const long long brow0 = (long long)(pr.routed ? e * pr.N : 0) + n0;
  auto b_at = [&](int n, int k) -> float {
    if (pr.ksplit) {
      const int j = k / pr.ksplit, kk = k % pr.ksplit;
      return Elem<T>::to_f(Bbase[((long long)j * pr.N + brow0 + n) * pr.ksplit + kk]);
    }
    return Elem<T>::to_f(Bbase[(brow0 + n) * pr.K + k]);
  };
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < pr.K; k0 += kSBK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid * 4 + i;          // 0..1023 over a 64 x 16 tile
      const int m = idx >> 4, k = idx & 15;
      As[k][m] = m < valid ? Elem<T>::to_f(A[(long long)m * pr.K + k0 + k]) : 0.f;
      Bs[k][m] = b_at(m, k0 + k);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kSBK; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { av[i] = As[k][ty * 4 + i]; bv[i] = Bs[k][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const T* bias = pr.bias ? reinterpret_cast<const T*>(pr.bias) + (long long)e * pr.bias_stride : nullptr;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = ty * 4 + i;
    if (m >= valid) continue;
    const long long grow = (long long)row0 + m;
    const float gate = pr.gate ? pr.gate[grow] : 1.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      float b = 0.f;
      if (bias)
        for (int br = 0; br < pr.bias_rows; ++br) b += Elem<T>::to_f(bias[(long long)br * pr.N + n]);
      const float u = acc[i][j] + b;
      if (pr.epi == 0)
        reinterpret_cast<T*>(pr.out)[grow * pr.ld_out + n] = Elem<T>::from_f(gelu_act<false>(u, a.act));
      else
        reinterpret_cast<T*>(pr.out)[grow * pr.ld_out + n] = Elem<T>::from_f(u * gate);
    }
  }
}

cudaError_t launch_gemm_simt(const GemmArgs& a, cudaStream_t s) {
  int maxn = 0;
  long long maxm = 0;
  for (int q = 0; q < a.nprob; ++q) {
    if (a.p[q].N > maxn) maxn = a.p[q].N;
    const long long m = a.p[q].routed ? a.r_max : a.p[q].M;
    if (m > maxm) maxm = m;
  }
  if (maxm == 0 || maxn == 0) return cudaSuccess;
  dim3 grid((maxn + kSBN - 1) / kSBN, (unsigned)((maxm + kSBM - 1) / kSBM), a.nprob);
  if (a.b16 && a.f16) gemm_simt_kernel<__half><<<grid, 256, 0, s>>>(a);
  else if (a.b16) gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a);
  else gemm_simt_kernel<float><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
