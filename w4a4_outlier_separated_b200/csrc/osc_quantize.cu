// OSC online quantization (one HBM pass over X): outlier extraction through the static
// suppression table, group amax, E8M0 shared exponent and E2M1 (or E4M3) encoding, written
// straight into the layouts the tcgen05 block-scaled MMA consumes.
//
// Method: the OSC page ("W4A4量化技术：OSC框架如何实现高效LLM部署", coreui.cn/article/2607942.html),
// §3.2 and Figure 2: for the table's channel of each group, copy the value into the
// high-precision buffer B and zero it, then microscale the zeroed group (a tighter scale).
// §4: the W2 fallback microscales to FP8 instead, with no separation.
//
// Work split: one thread owns 8 consecutive channels (one 16-byte load); the G/8 threads of
// a group reduce the amax with warp shuffles; a warp covers 256 consecutive channels of one
// row, so loads and the packed code stores are fully coalesced.
#include "osc_device.cuh"
#include "osc_internal.h"

namespace osc {

// Byte offset of the 32-bit word that holds scale slots [4*slot4, 4*slot4+4) of a row in
// the MMA scale layout: 512-byte atoms of 128 rows x 4 slots, row r of an atom at
// (r % 32) * 16 + (r / 32 % 4) * 4, atoms ordered by (row block, slot4).
__device__ __forceinline__ size_t scale_word_offset(int row, int slot4, int nslot4) {
  return ((size_t)(row >> 7) * nslot4 + slot4) * 512u + (size_t)((row & 31) * 16 + ((row >> 5) & 3) * 4);
}

__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;   // low nibble = lo, high nibble = hi
}

__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;   // low byte = lo, high byte = hi
}

// Codes whose magnitude rounds to zero take the sign of the input (so -0.1 -> 0x8 / 0x80),
// whatever the conversion instruction does with negative values that round to zero.
__device__ __forceinline__ uint32_t e2m1_fix_zero_sign(uint32_t p, const uint32_t (&w)[4]) {
  uint32_t nz = (p | (p >> 1) | (p >> 2)) & 0x11111111u;
  uint32_t zpos = ((~nz) & 0x11111111u) << 3;
  uint32_t s = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) s |= (((w[j] >> 12) & 0x8u) | ((w[j] >> 24) & 0x80u)) << (8 * j);
  return (p & ~zpos) | (s & zpos);
}

__device__ __forceinline__ uint32_t e4m3_fix_zero_sign(uint32_t h, uint32_t w0, uint32_t w1) {
  uint32_t m = h & 0x7F7F7F7Fu;
  uint32_t nz = ((m + 0x7F7F7F7Fu) | m) & 0x80808080u;
  uint32_t z = (~nz) & 0x80808080u;
  uint32_t s = ((w0 >> 8) & 0x80u) | ((w0 >> 16) & 0x8000u) | ((w1 << 8) & 0x800000u) | (w1 & 0x80000000u);
  return (h & ~z) | (s & z);
}

// Stage one table in shared memory with each entry's column in B (exclusive scan over the
// valid entries). Entries >= G, and entries beyond K_L columns, are reported and dropped.
template <int G>
__device__ __forceinline__ int stage_table(const int8_t* __restrict__ L, int Kg, int K_L, int8_t* Ls,
                                           int16_t* pos, int* s_warp, int* status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (Kg + 255) / 256;
  int local = 0;
  for (int i = tid * per; i < min(Kg, tid * per + per); ++i) {
    int v = L[i];
    if (v >= G) { record_status(status, DEV_BAD_TABLE); v = -1; }
    Ls[i] = (int8_t)v;
    local += (v >= 0);
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int base = 0, total = 0;
  for (int w = 0; w < 8; ++w) { if (w < warp) base += s_warp[w]; total += s_warp[w]; }
  int run = base + incl - local;
  for (int i = tid * per; i < min(Kg, tid * per + per); ++i) {
    if (Ls[i] >= 0) {
      if (run >= K_L) { record_status(status, DEV_BAD_TABLE); Ls[i] = -1; }
      pos[i] = (int16_t)run;
      ++run;
    }
  }
  __syncthreads();
  return total < K_L ? total : K_L;
}

// One 16-byte chunk (8 channels k0..k0+7 of one row): extraction through the staged table,
// group amax over the G/8 lanes of the group, E8M0 exponent, E2M1/E4M3 codes and the scale
// word. Called by all 32 lanes of a warp together (the shuffles span the warp).
template <int G, bool FP8, bool TABLE>
__device__ __forceinline__ void quant_chunk(uint32_t (&w)[4], int row, int kc, int K, const int8_t* Ls,
                                            const int16_t* pos, int count, int K_L, uint16_t* __restrict__ B,
                                            uint8_t* __restrict__ Q, uint8_t* __restrict__ S) {
  constexpr int V = FP8 ? 32 : (G == 16 ? 16 : 32);      // scale slot width
  constexpr int GL = (FP8 ? 32 : G) / 8;                   // lanes per amax group
  constexpr int EMAX = FP8 ? 8 : 2;
  const int k0 = kc * 8;
  if constexpr (TABLE) {
    const int g = k0 / G;
    const int l = Ls[g];
    const int off = l - (k0 % G);
    if (l >= 0 && off >= 0 && off < 8) {
      const uint32_t sh = (off & 1) * 16;
      B[(size_t)row * K_L + pos[g]] = (uint16_t)(w[off >> 1] >> sh);
      w[off >> 1] &= ~(0xFFFFu << sh);           // the slot becomes +0
    }
    if (kc == 0)
      for (int i = count; i < K_L; ++i) B[(size_t)row * K_L + i] = 0;
  }

  // group amax on the bf16 magnitude bits (monotone for finite values)
  uint32_t am = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) am = max(am, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
#pragma unroll
  for (int o = 1; o < GL; o <<= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
  const int eb = (int)(am >> 7);
  const int e = (eb == 0) ? -127 : max(eb - 127 - EMAX, -127);
  const float f = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e, exact

  float x[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(w[j] << 16) * f;
    x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u) * f;
  }
  if constexpr (!FP8) {
    uint32_t q = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) q |= cvt_e2m1x2(x[2 * j], x[2 * j + 1]) << (8 * j);
    q = e2m1_fix_zero_sign(q, w);
    reinterpret_cast<uint32_t*>(Q)[(size_t)row * (K / 8) + kc] = q;
  } else {
    uint32_t h0 = cvt_e4m3x2(x[0], x[1]) | (cvt_e4m3x2(x[2], x[3]) << 16);
    uint32_t h1 = cvt_e4m3x2(x[4], x[5]) | (cvt_e4m3x2(x[6], x[7]) << 16);
    h0 = e4m3_fix_zero_sign(h0, w[0], w[1]);
    h1 = e4m3_fix_zero_sign(h1, w[2], w[3]);
    reinterpret_cast<uint2*>(Q)[(size_t)row * (K / 8) + kc] = make_uint2(h0, h1);
  }

  // scale codes: the lane that starts a 4-slot word gathers it and stores 32 bits
  const uint32_t code = (uint32_t)(e + 127);
  constexpr int SL = V / 8;                   // lanes per slot
  const uint32_t c1 = __shfl_down_sync(0xffffffffu, code, SL);
  const uint32_t c2 = __shfl_down_sync(0xffffffffu, code, 2 * SL);
  const uint32_t c3 = __shfl_down_sync(0xffffffffu, code, 3 * SL);
  if (kc % (4 * SL) == 0) {
    const int slot4 = k0 / (4 * V);
    *reinterpret_cast<uint32_t*>(S + scale_word_offset(row, slot4, K / V / 4)) =
        code | (c1 << 8) | (c2 << 16) | (c3 << 24);
  }
}

template <int G, bool FP8, bool TABLE>
__global__ void __launch_bounds__(256) quantize_kernel(QuantParams p) {
  constexpr int V = FP8 ? 32 : (G == 16 ? 16 : 32);
  extern __shared__ __align__(16) unsigned char qsm[];
  int8_t* Ls = reinterpret_cast<int8_t*>(qsm);
  int16_t* pos = reinterpret_cast<int16_t*>(qsm + ((p.Kg + 15) & ~15));
  __shared__ int s_warp[8];
  const int K = p.K, M = p.M;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int count = 0;
  if constexpr (TABLE) count = stage_table<G>(p.L, p.Kg, p.K_L, Ls, pos, s_warp, p.status);

  const int cpr = K / 8;                        // 16-byte chunks per row
  const long long total = (long long)M * cpr;   // a multiple of 32 (K % 256 == 0)
  const long long gwarp = (long long)blockIdx.x * 8 + warp;
  const long long nwarps = (long long)gridDim.x * 8;
  constexpr int U = 2;                          // two independent 16-byte loads in flight per thread
  for (long long base = gwarp * 32 * U; base < total; base += nwarps * 32 * U) {
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (base + u * 32 < total) raw[u] = __ldcs(reinterpret_cast<const uint4*>(p.X) + base + u * 32 + lane);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (base + u * 32 >= total) break;          // warp-uniform
      const long long c = base + u * 32 + lane;
      const int row = (int)(c / cpr);
      const int kc = (int)(c - (long long)row * cpr);
      uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
      quant_chunk<G, FP8, TABLE>(w, row, kc, K, Ls, pos, count, p.K_L, p.B, p.Q, p.S);
    }
  }

  // rows between M and the next multiple of 128 hold zero scales (2^-127)
  const int nslot4 = K / V / 4;
  const int mpad = (M + 127) / 128 * 128;
  const long long npad = (long long)(mpad - M) * nslot4;
  for (long long i = (long long)blockIdx.x * 256 + tid; i < npad; i += (long long)gridDim.x * 256) {
    const int row = M + (int)(i / nslot4);
    const int s4 = (int)(i % nslot4);
    *reinterpret_cast<uint32_t*>(p.S + scale_word_offset(row, s4, nslot4)) = 0u;
  }
}

// Grouped (MoE) form: each CTA takes whole 128-row blocks of the padded row space; a block
// belongs to one expert, whose table is staged once. Rows past the expert's token count are
// padding and are written as zeros (codes 0, scale 2^-127, B 0).
template <int G>
__global__ void __launch_bounds__(256) quantize_grouped_kernel(GroupedQuantParams p) {
  extern __shared__ __align__(16) unsigned char qsm[];
  int8_t* Ls = reinterpret_cast<int8_t*>(qsm);
  int16_t* pos = reinterpret_cast<int16_t*>(qsm + ((p.Kg + 15) & ~15));
  __shared__ int s_warp[8];
  const int K = p.K;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cpr = K / 8;
  const int nblocks = p.Mp / 128;
  for (int mb = blockIdx.x; mb < nblocks; mb += gridDim.x) {
    const int e = __ldg(p.mblock_expert + mb);
    const int cnt = __ldg(p.off + e + 1) - __ldg(p.off + e);
    const int src0 = __ldg(p.off + e);
    const int prow0 = __ldg(p.poff + e);
    __syncthreads();                               // the previous block's table readers are done
    const int count = stage_table<G>(p.L + (size_t)e * p.Kg, p.Kg, p.K_L, Ls, pos, s_warp, p.status);
    const int total = 128 * cpr;                   // chunks in this block, a multiple of 32
    for (int base = warp * 64; base < total; base += 8 * 64) {
      uint4 raw[2];
      int rows[2], kcs[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = base + u * 32 + lane;
        rows[u] = mb * 128 + c / cpr;
        kcs[u] = c % cpr;
        const int local = rows[u] - prow0;
        raw[u] = make_uint4(0u, 0u, 0u, 0u);
        if (base + u * 32 < total && local < cnt)
          raw[u] = __ldcs(reinterpret_cast<const uint4*>(p.X + (size_t)(src0 + local) * K) + kcs[u]);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (base + u * 32 >= total) break;         // warp-uniform
        uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
        quant_chunk<G, false, true>(w, rows[u], kcs[u], K, Ls, pos, count, p.K_L, p.B, p.Q, p.S);
      }
    }
  }
}

template <int G, bool FP8, bool TABLE>
static cudaError_t launch_quant(const QuantParams& p, int grid, cudaStream_t s) {
  size_t smem = TABLE ? (size_t)((p.Kg + 15) & ~15) + (size_t)p.Kg * 2 : 0;
  quantize_kernel<G, FP8, TABLE><<<grid, 256, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantParams& p, bool fp8, int num_sms, cudaStream_t s) {
  const long long chunks = (long long)p.M * (p.K / 8);
  long long want = (chunks + 511) / 512;                 // 256 threads x 2 chunks
  const long long pad_words = (long long)((p.M + 127) / 128 * 128 - p.M) * (p.K / 128);
  want = std::max(want, (pad_words + 255) / 256);
  const int grid = (int)std::min<long long>(std::max<long long>(want, 1), (long long)num_sms * 8);
  const bool table = p.L != nullptr;
  if (fp8) return launch_quant<32, true, false>(p, grid, s);
  switch (p.G) {
    case 16: return table ? launch_quant<16, false, true>(p, grid, s) : launch_quant<16, false, false>(p, grid, s);
    case 32: return table ? launch_quant<32, false, true>(p, grid, s) : launch_quant<32, false, false>(p, grid, s);
    case 64: return table ? launch_quant<64, false, true>(p, grid, s) : launch_quant<64, false, false>(p, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize_grouped(const GroupedQuantParams& p, int num_sms, cudaStream_t s) {
  const int nblocks = p.Mp / 128;
  if (nblocks == 0) return cudaSuccess;
  const int grid = std::min(nblocks, num_sms * 4);
  const size_t smem = (size_t)((p.Kg + 15) & ~15) + (size_t)p.Kg * 2;
  switch (p.G) {
    case 16: quantize_grouped_kernel<16><<<grid, 256, smem, s>>>(p); break;
    case 32: quantize_grouped_kernel<32><<<grid, 256, smem, s>>>(p); break;
    case 64: quantize_grouped_kernel<64><<<grid, 256, smem, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// W_L (§3.2/§3.3): the bf16 weight columns of the table's channels, one contiguous
// N x K_L block; pad columns are zero.
__global__ void __launch_bounds__(256) gather_wl_kernel(const uint16_t* __restrict__ W, int N, int K, int G,
                                                        const int8_t* __restrict__ L, int Kg, int K_L,
                                                        uint16_t* __restrict__ WL, int* status) {
  extern __shared__ int chan[];          // K_L entries: source channel, or -1 for pad
  if (threadIdx.x == 0) {
    int c = 0;
    for (int k = 0; k < Kg; ++k) {
      int v = L[k];
      if (v >= G) { record_status(status, DEV_BAD_TABLE); continue; }
      if (v < 0) continue;
      if (c >= K_L) { record_status(status, DEV_BAD_TABLE); break; }
      chan[c++] = k * G + v;
    }
    for (; c < K_L; ++c) chan[c] = -1;
  }
  __syncthreads();
  const long long total = (long long)N * K_L;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(i / K_L), j = (int)(i % K_L);
    const int ch = chan[j];
    WL[i] = ch >= 0 ? W[(size_t)n * K + ch] : (uint16_t)0;
  }
}

cudaError_t launch_gather_wl(const uint16_t* W, int N, int K, int G, const int8_t* L, int K_L, uint16_t* WL,
                             int* status, int num_sms, cudaStream_t s) {
  if (K_L == 0 || N == 0) return cudaSuccess;
  long long total = (long long)N * K_L;
  int grid = (int)std::min<long long>((total + 255) / 256, (long long)num_sms * 4);
  gather_wl_kernel<<<grid, 256, (size_t)K_L * sizeof(int), s>>>(W, N, K, G, L, K / G, K_L, WL, status);
  return cudaGetLastError();
}

}  // namespace osc
