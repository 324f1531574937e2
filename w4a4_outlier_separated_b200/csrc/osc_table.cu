// Offline suppression-table build on the GPU: Algorithm 1 of the OSC page
// ("W4A4量化技术：OSC框架如何实现高效LLM部署", coreui.cn/article/2607942.html, §3.1), for one
// (position, layer) given its S x K calibration activations.
//
// find_consistent_outlier is left undefined by the page; the rule used here: for each
// calibration token the group's outlier event is the channel with the largest |x| (lowest
// channel on ties), counted only when G * |x_max| >= alpha * sum_j |x_j| and |x_max| > 0; the
// sum runs in fp32 in ascending channel order and the comparison in fp64, so the decision is
// reproducible bit for bit. The channel with the most events wins (lowest on ties) when it
// has at least min_hits events; otherwise the entry is -1. Counting is integer, so the table
// does not depend on the order in which tokens are visited.
//
// One CTA per channel group; threads stride over tokens; a shared histogram of G counters.
//
// The clustering density of §2.2 uses the same event: over a set of tokens, N_total(k) counts
// group k's events and N_hit(k) those whose channel is the table's entry L[k]; the ratio
// C_k = N_hit / N_total, averaged over the groups with events, selects the tier of §2.3.
#include "osc_device.cuh"
#include "osc_internal.h"

namespace osc {

// One token's group of G bf16 values at xg (16-byte aligned): the channel of largest |x|
// (lowest on ties, compared on the magnitude bits) and whether it is an outlier event.
// Channels whose bit is set in `masked` count as zero (they were protected in an earlier
// round of a multi-entry table build).
template <int G>
__device__ __forceinline__ bool group_event(const uint16_t* xg, float alpha, int* j_out, uint64_t masked = 0) {
  const uint4* src = reinterpret_cast<const uint4*>(xg);
  float s = 0.0f;
  uint32_t best = 0;
  int jb = 0;
#pragma unroll
  for (int v = 0; v < G / 8; ++v) {
    const uint4 r = __ldg(src + v);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      uint32_t mag = (h & 1) ? (w[h >> 1] >> 16) & 0x7FFFu : w[h >> 1] & 0x7FFFu;
      if ((masked >> (v * 8 + h)) & 1u) mag = 0u;
      s += __uint_as_float(mag << 16);
      if (mag > best) { best = mag; jb = v * 8 + h; }
    }
  }
  *j_out = jb;
  const double amax = (double)__uint_as_float(best << 16);
  return best != 0u && (double)G * amax >= (double)alpha * (double)s;
}

// R rounds (R protected channels at most): round r repeats the count with the channels of the
// earlier rounds read as zero, which is what extraction leaves of the group; once a round finds
// no channel the later ones find none either.
template <int G>
__global__ void __launch_bounds__(256) build_table_kernel(TableParams p) {
  __shared__ int hist[G];
  __shared__ int s_pick;
  const int k = blockIdx.x;
  uint64_t masked = 0;
  for (int r = 0; r < p.R; ++r) {
    for (int j = threadIdx.x; j < G; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < p.S; t += blockDim.x) {
      int jb;
      if (group_event<G>(p.X + (size_t)t * p.K + (size_t)k * G, p.alpha, &jb, masked)) atomicAdd(&hist[jb], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int js = 0;
      for (int j = 1; j < G; ++j)
        if (hist[j] > hist[js]) js = j;
      s_pick = (hist[js] > 0 && hist[js] >= p.min_hits) ? js : -1;
      p.L[(size_t)k * p.R + r] = (int8_t)s_pick;
    }
    __syncthreads();
    const int pick = s_pick;
    if (pick >= 0) masked |= 1ull << pick;
    __syncthreads();                         // s_pick is read by all before the next round
  }
}

// One CTA per group: the group's event and hit counts over the S tokens.
template <int G>
__global__ void __launch_bounds__(256) density_kernel(DensityParams p) {
  __shared__ int cnt[2];
  const int k = blockIdx.x;
  if (threadIdx.x < 2) cnt[threadIdx.x] = 0;
  const int l = p.L[k];
  if (threadIdx.x == 0 && l >= G) record_status(p.status, DEV_BAD_TABLE);   // never matches a channel
  __syncthreads();
  int hit = 0, tot = 0;
  for (int t = threadIdx.x; t < p.S; t += blockDim.x) {
    int jb;
    if (group_event<G>(p.X + (size_t)t * p.K + (size_t)k * G, p.alpha, &jb)) {
      ++tot;
      hit += (jb == l);
    }
  }
  if (tot) {
    atomicAdd(&cnt[0], hit);
    atomicAdd(&cnt[1], tot);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    p.n_hit[k] = cnt[0];
    p.n_total[k] = cnt[1];
  }
}

cudaError_t launch_density(const DensityParams& p, cudaStream_t s) {
  const int Kg = p.K / p.G;
  if (Kg == 0) return cudaSuccess;
  switch (p.G) {
    case 16: density_kernel<16><<<Kg, 256, 0, s>>>(p); break;
    case 32: density_kernel<32><<<Kg, 256, 0, s>>>(p); break;
    case 64: density_kernel<64><<<Kg, 256, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_build_table(const TableParams& p, int num_sms, cudaStream_t s) {
  (void)num_sms;
  const int Kg = p.K / p.G;
  if (Kg == 0) return cudaSuccess;
  switch (p.G) {
    case 16: build_table_kernel<16><<<Kg, 256, 0, s>>>(p); break;
    case 32: build_table_kernel<32><<<Kg, 256, 0, s>>>(p); break;
    case 64: build_table_kernel<64><<<Kg, 256, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace osc
