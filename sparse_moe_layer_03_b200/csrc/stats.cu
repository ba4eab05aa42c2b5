// Expert-selection statistics.
//
// Expert-selection frequency per label: the statistic behind the expert
// specialisation heat maps of "Scaling Diffusion Transformers to 16 Billion
// Parameters" (selection frequency by image class, by spatial position and by
// denoising timestep).  One thread per token; each slot's (label, expert)
// key is merged across the warp (match.any) before one global atomic per
// distinct key.  Integer counts, so the order of the atomics does not matter.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kFreqThreads = 256;

__global__ void __launch_bounds__(kFreqThreads) frequency_kernel(FreqArgs a) {
  const int t = blockIdx.x * kFreqThreads + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const bool valid = t < a.T;
  int label = -1;
  if (valid) {
    label = a.labels ? a.labels[t / a.L] : t % a.L;
    if (label < 0 || label >= a.n_labels) {
      set_status(a.status, DEV_BAD_INDEX, 400);
      label = -1;
    }
  }
  const int ns = label >= 0 ? (a.n_sel ? a.n_sel[t] : a.K) : 0;
  for (int k = 0; k < a.Kmax; ++k) {     // the same trip count in every lane
    int key = -1;
    if (k < ns) {
      const int e = a.topk_idx[(size_t)t * a.Kmax + k];
      if (e >= a.E) set_status(a.status, DEV_BAD_INDEX, 401);
      else if (e >= 0) key = label * a.E + e;
    }
    const unsigned same = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && lane == __ffs(same) - 1) atomicAdd(&a.hist[key], __popc(same));
  }
}

cudaError_t launch_frequency(const FreqArgs& a, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(a.hist, 0, (size_t)a.n_labels * a.E * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  if (a.T == 0) return cudaSuccess;
  frequency_kernel<<<(a.T + kFreqThreads - 1) / kFreqThreads, kFreqThreads, 0, s>>>(a);
  return cudaGetLastError();
}

// Balance-loss statistics ("MOE-DIT", eq. L_balance).  The loss is a function
// of two per-expert sums over the tokens, counts_i = sum_t I(t,i) and
// s_i = sum_t P[t,i]; over a batch split between ranks both are sums of the
// ranks' own, so one all-reduce of the 2E values [counts, s] gives the loss of
// the whole batch: L = alpha sum_i (E / (K T)) counts_i (s_i / T), T = all tokens.
// Counts travel as fp64 (exact below 2^53).
__global__ void balance_stats_kernel(const int32_t* counts, const double* score_sum, int E, double* stats) {
  const int i = threadIdx.x;
  if (i < E) {
    stats[i] = (double)counts[i];
    stats[E + i] = score_sum[i];
  }
}

// One warp; the terms are added in a fixed tree order (bit-reproducible), as in
// the router's own finalize.
__global__ void balance_loss_from_stats_kernel(const double* stats, int E, int K, long long T_total, float alpha,
                                               float* aux_loss) {
  const int i = threadIdx.x;
  double term = 0.0;
  if (i < E && T_total > 0) {
    const double T = (double)T_total;
    term = ((double)E / ((double)K * T)) * stats[i] * (stats[E + i] / T);
  }
  for (int o = 16; o > 0; o >>= 1) term += __shfl_down_sync(0xffffffffu, term, o);
  if (i == 0) *aux_loss = (float)(alpha * term);
}

cudaError_t launch_balance_stats(const int32_t* counts, const double* score_sum, int E, double* stats,
                                 cudaStream_t s) {
  balance_stats_kernel<<<1, 32, 0, s>>>(counts, score_sum, E, stats);
  return cudaGetLastError();
}

cudaError_t launch_balance_loss_from_stats(const double* stats, int E, int K, long long T_total, float alpha,
                                           float* aux_loss, cudaStream_t s) {
  balance_loss_from_stats_kernel<<<1, 32, 0, s>>>(stats, E, K, T_total, alpha, aux_loss);
  return cudaGetLastError();
}

}  // namespace moe
