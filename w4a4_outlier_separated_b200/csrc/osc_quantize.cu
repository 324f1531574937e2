// OSC online quantization (one HBM pass over X): outlier extraction through the static
// suppression table, group amax, E8M0 shared exponent and E2M1 (or E4M3) encoding, written
// straight into the layouts the tcgen05 block-scaled MMA consumes.
//
// Method: the OSC page ("W4A4量化技术：OSC框架如何实现高效LLM部署", coreui.cn/article/2607942.html),
// §3.2 and Figure 2: for the table's channel of each group, copy the value into the
// high-precision buffer B and zero it, then microscale the zeroed group (a tighter scale).
// §4: the W2 fallback microscales to FP8 instead, with no separation.
//
// Work split: a warp owns one 256-channel segment over a few rows; each lane owns 8
// consecutive channels (one 16-byte load per row) and works out once which of them is a table
// channel; the G/8 lanes of a group reduce the amax with warp shuffles. Loads and the packed
// code stores are fully coalesced (512 and 128 contiguous bytes per warp and row).
#include "osc_device.cuh"
#include "osc_internal.h"

namespace osc {

// Byte offset of the 32-bit word that holds scale slots [4*slot4, 4*slot4+4) of a row in
// the MMA scale layout: 512-byte atoms of 128 rows x 4 slots, row r of an atom at
// (r % 32) * 16 + (r / 32 % 4) * 4, atoms ordered by (row block, slot4).
__device__ __forceinline__ size_t scale_word_offset(int row, int slot4, int nslot4) {
  return ((size_t)(row >> 7) * nslot4 + slot4) * 512u + (size_t)((row & 31) * 16 + ((row >> 5) & 3) * 4);
}

// Eight E2M1 codes from eight fp32 values (already scaled by 2^-e), packed low nibble first.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&x)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 a, b, c, d;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 a, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 d, %8, %7;\n\t"
      "mov.b32 %0, {a, b, c, d};\n\t}"
      : "=r"(r) : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
  return r;
}

// Four E4M3 codes, low byte first.
__device__ __forceinline__ uint32_t cvt_e4m3x4(float x0, float x1, float x2, float x3) {
  uint32_t r;
  asm("{\n\t.reg .b16 a, b;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 a, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 b, %4, %3;\n\t"
      "mov.b32 %0, {a, b};\n\t}"
      : "=r"(r) : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
  return r;
}

// What one lane needs to know about its 8 channels of a 256-channel segment, independent of
// the row: whether the segment slot holds the table's channel, which of the 8 it is, and its
// column in B. Computed once per warp task from the table with ballots (no shared memory).
struct LaneTable {
  int has;     // 1 if one of this lane's 8 channels is the group's table channel
  int eidx;    // which of the 8
  int pos;     // its column in B
  int count;   // valid entries in the whole table (min K_L)
};

template <int G>
__device__ __forceinline__ LaneTable lane_table(const int8_t* __restrict__ L, int Kg, int K_L, int seg, int lane,
                                                int* status) {
  constexpr int LPG = G / 8;                              // lanes per group
  const int g0 = seg * 256 / G;                           // first group of the segment
  const int glane = g0 + lane / LPG;
  const unsigned full = 0xffffffffu;
  int before = 0;
  for (int j = 0; j < g0; j += 32) {
    const int k = j + lane;
    int v = (k < g0) ? (int)L[k] : -1;
    before += __popc(__ballot_sync(full, v >= 0 && v < G));
  }
  int l = L[glane];
  if (l >= G) { if (lane % LPG == 0) record_status(status, DEV_BAD_TABLE); l = -1; }
  const unsigned firsts = __ballot_sync(full, (lane % LPG == 0) && l >= 0);
  const int fl = (lane / LPG) * LPG;                      // first lane of my group
  LaneTable t;
  t.pos = before + __popc(firsts & ((1u << fl) - 1u));
  t.eidx = l - (lane % LPG) * 8;
  t.has = (l >= 0 && t.eidx >= 0 && t.eidx < 8) ? 1 : 0;
  if (t.has && t.pos >= K_L) { record_status(status, DEV_BAD_TABLE); t.has = 0; }
  t.count = 0;
  if (seg == 0) {                                         // only segment 0 writes the pad columns
    int c = 0;
    for (int j = 0; j < Kg; j += 32) {
      const int k = j + lane;
      int v = (k < Kg) ? (int)L[k] : -1;
      c += __popc(__ballot_sync(full, v >= 0 && v < G));
    }
    t.count = c < K_L ? c : K_L;
  }
  return t;
}

// One row of one lane: extraction, group amax (G/8 lanes), exponent, codes, scale word.
// All 32 lanes of the warp call it together (shuffles).
template <int G, bool FP8, bool TABLE>
__device__ __forceinline__ void quant_row(uint4 raw, int row, int seg, int lane, int K, const LaneTable& t, int K_L,
                                          uint16_t* __restrict__ B, uint8_t* __restrict__ Q, uint8_t* __restrict__ S,
                                          bool store_q) {
  constexpr int V = FP8 ? 32 : (G == 16 ? 16 : 32);      // scale slot width
  constexpr int GL = (FP8 ? 32 : G) / 8;                   // lanes per amax group
  constexpr int EMAX = FP8 ? 8 : 2;
  uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  if constexpr (TABLE) {
    if (t.has) {
      const int j = t.eidx >> 1;
      const uint32_t sh = (t.eidx & 1) * 16;
      if (store_q) B[(size_t)row * K_L + t.pos] = (uint16_t)(w[j] >> sh);
      w[j] &= ~(0xFFFFu << sh);                  // the slot becomes +0
    }
    if (store_q && seg == 0 && lane == 0)
      for (int i = t.count; i < K_L; ++i) B[(size_t)row * K_L + i] = 0;
  }
  // amax over the magnitudes: for finite bf16 values |x| orders like its 15 low bits
  const uint32_t a0 = w[0] & 0x7FFF7FFFu, a1 = w[1] & 0x7FFF7FFFu, a2 = w[2] & 0x7FFF7FFFu, a3 = w[3] & 0x7FFF7FFFu;
  uint32_t mm = __vmaxu2(__vmaxu2(a0, a1), __vmaxu2(a2, a3));
  uint32_t am = max(mm & 0xFFFFu, mm >> 16);
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
  const size_t chunk = (size_t)row * (K / 8) + seg * 32 + lane;
  if constexpr (!FP8) {
    // the conversion keeps the sign of values that round to zero (-0.1 -> 0x8), as the
    // element rule requires; the every-bf16-value parity tests pin that behaviour
    uint32_t q = cvt_e2m1x8(x);
    if (store_q) reinterpret_cast<uint32_t*>(Q)[chunk] = q;
  } else {
    const uint32_t h0 = cvt_e4m3x4(x[0], x[1], x[2], x[3]);
    const uint32_t h1 = cvt_e4m3x4(x[4], x[5], x[6], x[7]);
    if (store_q) reinterpret_cast<uint2*>(Q)[chunk] = make_uint2(h0, h1);
  }
  // the lane that starts a 4-slot word gathers it and stores 32 bits
  const uint32_t code = (uint32_t)(e + 127);
  constexpr int SL = V / 8;                   // lanes per slot
  const uint32_t c1 = __shfl_down_sync(0xffffffffu, code, SL);
  const uint32_t c2 = __shfl_down_sync(0xffffffffu, code, 2 * SL);
  const uint32_t c3 = __shfl_down_sync(0xffffffffu, code, 3 * SL);
  if (lane % (4 * SL) == 0) {
    const int slot4 = (seg * 256 + lane * 8) / (4 * V);
    *reinterpret_cast<uint32_t*>(S + scale_word_offset(row, slot4, K / V / 4)) =
        code | (c1 << 8) | (c2 << 16) | (c3 << 24);
  }
}

constexpr int QROWS = 8;   // rows per dense warp task (divides 128: a task never leaves a 128-row block)
constexpr int GROWS = 8;   // rows per grouped warp task
constexpr int MAX_KG = 1024;

// Dense form. The CTA stages the table once: each entry's channel and its column in B
// (exclusive count of the valid entries before it). A warp task is one 256-channel segment x
// QROWS rows; its lanes read their table facts from shared memory. Rows from M up to the
// next multiple of 128 only get zero scales.
template <int G, bool FP8, bool TABLE>
__global__ void __launch_bounds__(256) quantize_kernel(QuantParams p) {
  __shared__ int8_t s_l[TABLE ? MAX_KG : 1];
  __shared__ int16_t s_pos[TABLE ? MAX_KG : 1];
  __shared__ int s_warp[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int count = 0;
  if constexpr (TABLE) {
    const int per = (p.Kg + 255) / 256;
    const int i0 = threadIdx.x * per, i1 = min(p.Kg, i0 + per);
    int local = 0;
    for (int i = i0; i < i1; ++i) {
      int v = p.L[i];
      if (v >= G) { record_status(p.status, DEV_BAD_TABLE); v = -1; }
      s_l[i] = (int8_t)v;
      local += v >= 0;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int run = incl - local;
    for (int w = 0; w < 8; ++w) { if (w < warp) run += s_warp[w]; count += s_warp[w]; }
    for (int i = i0; i < i1; ++i)
      if (s_l[i] >= 0) {
        if (run >= p.K_L) { record_status(p.status, DEV_BAD_TABLE); s_l[i] = -1; }
        s_pos[i] = (int16_t)run++;
      }
    count = min(count, p.K_L);
    __syncthreads();
  }
  const int nseg = p.K / 256;
  const int mpad = (p.M + 127) / 128 * 128;
  const int tasks = nseg * (mpad / QROWS);
  const int cpr = p.K / 8;
  for (int task = blockIdx.x * 8 + warp; task < tasks; task += gridDim.x * 8) {
    const int seg = task % nseg;
    const int r0 = (task / nseg) * QROWS;
    LaneTable t{};
    if constexpr (TABLE) {
      const int k0 = seg * 256 + lane * 8;
      const int g = k0 / G;
      const int l = s_l[g];
      t.eidx = l - (k0 % G);
      t.has = (l >= 0 && t.eidx >= 0 && t.eidx < 8) ? 1 : 0;
      t.pos = s_pos[g];
      t.count = count;
    }
    const uint4* src = reinterpret_cast<const uint4*>(p.X) + seg * 32 + lane;
    uint4 raw[QROWS];                               // all of the task's loads in flight at once
#pragma unroll
    for (int u = 0; u < QROWS; ++u) {
      const int r = r0 + u;
      raw[u] = r < p.M ? __ldcs(src + (size_t)r * cpr) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < QROWS; ++u) {
      const int r = r0 + u;
      quant_row<G, FP8, TABLE>(raw[u], r, seg, lane, p.K, t, p.K_L, p.B, p.Q, p.S, r < p.M);
    }
  }
}

// Grouped (MoE) form over the padded row space: a task's rows lie in one 128-row block, which
// belongs to one expert; rows past the expert's token count are padding and come out as zeros.
template <int G>
__global__ void __launch_bounds__(256) quantize_grouped_kernel(GroupedQuantParams p) {
  const int lane = threadIdx.x & 31;
  const int nseg = p.K / 256;
  const int tasks = nseg * (p.Mp / GROWS);
  const int cpr = p.K / 8;
  for (int task = blockIdx.x * 8 + (threadIdx.x >> 5); task < tasks; task += gridDim.x * 8) {
    const int seg = task % nseg;
    const int r0 = (task / nseg) * GROWS;
    const int e = __ldg(p.mblock_expert + r0 / 128);
    const int src0 = __ldg(p.off + e);
    const int cnt = __ldg(p.off + e + 1) - src0;
    const int prow0 = __ldg(p.poff + e);
    const LaneTable t = lane_table<G>(p.L + (size_t)e * p.Kg, p.Kg, p.K_L, seg, lane, p.status);
    const uint4* src = reinterpret_cast<const uint4*>(p.X) + seg * 32 + lane;
    uint4 raw[GROWS];
#pragma unroll
    for (int u = 0; u < GROWS; ++u) {
      const int local = r0 + u - prow0;
      raw[u] = local < cnt ? __ldcs(src + (size_t)(src0 + local) * cpr) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < GROWS; ++u)
      quant_row<G, false, true>(raw[u], r0 + u, seg, lane, p.K, t, p.K_L, p.B, p.Q, p.S, true);
  }
}

template <int G, bool FP8, bool TABLE>
static cudaError_t launch_quant(const QuantParams& p, int grid, cudaStream_t s) {
  quantize_kernel<G, FP8, TABLE><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

static int quant_grid(long long tasks, int num_sms) {
  const long long want = (tasks + 7) / 8;
  return (int)std::max<long long>(1, std::min<long long>(want, (long long)num_sms * 8));
}

cudaError_t launch_quantize(const QuantParams& p, bool fp8, int num_sms, cudaStream_t s) {
  const int grid = quant_grid((long long)(p.K / 256) * ((p.M + 127) / 128 * 128 / QROWS), num_sms);
  if (p.L != nullptr && p.Kg > MAX_KG) return cudaErrorInvalidValue;
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
  if (p.Mp == 0) return cudaSuccess;
  const int grid = quant_grid((long long)(p.K / 256) * (p.Mp / GROWS), num_sms);
  switch (p.G) {
    case 16: quantize_grouped_kernel<16><<<grid, 256, 0, s>>>(p); break;
    case 32: quantize_grouped_kernel<32><<<grid, 256, 0, s>>>(p); break;
    case 64: quantize_grouped_kernel<64><<<grid, 256, 0, s>>>(p); break;
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
