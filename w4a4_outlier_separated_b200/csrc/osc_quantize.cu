// OSC online quantization (one HBM pass over X): outlier extraction through the static
// suppression table, group amax, E8M0 shared exponent and E2M1 (or E4M3) encoding, written
// straight into the layouts the tcgen05 block-scaled MMA consumes.
//
// Method: the OSC page ("W4A4量化技术：OSC框架如何实现高效LLM部署", coreui.cn/article/2607942.html),
// §3.2 and Figure 2: for the table's channel of each group, copy the value into the
// high-precision buffer B and zero it, then microscale the zeroed group (a tighter scale).
// §4: the W2 fallback microscales to FP8 instead, with no separation.
//
// Work split: a thread owns a 32-channel block of a row (four 16-byte loads, 32 codes stored
// as one 16-byte write), so the block amax needs no cross-thread reduction (G = 64 pairs two
// neighbouring threads); the table sits in shared memory once per CTA. Neighbouring threads
// hold neighbouring blocks, so a warp's loads and stores cover contiguous runs of each row.
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
__device__ __forceinline__ uint32_t cvt_e2m1x8(float x0, float x1, float x2, float x3, float x4, float x5,
                                               float x6, float x7) {
  uint32_t r;
  asm("{\n\t.reg .b8 a, b, c, d;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 a, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 d, %8, %7;\n\t"
      "mov.b32 %0, {a, b, c, d};\n\t}"
      : "=r"(r) : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
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

__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Shared exponent e (unbiased) from the largest magnitude bits of a block: floor(log2 amax)
// - emax, clamped at -127 (an all-zero or subnormal-only block gets -127).
template <int EMAX>
__device__ __forceinline__ int shared_exp(uint32_t am) {
  const int eb = (int)(am >> 7);
  return (eb == 0) ? -127 : max(eb - 127 - EMAX, -127);
}

// Largest |x| bits over words [J0, J0+NW) of a 32-element block (bf16 pairs).
template <int J0, int NW>
__device__ __forceinline__ uint32_t block_amax(const uint32_t (&w)[16]) {
  uint32_t m = w[J0] & 0x7FFF7FFFu;
#pragma unroll
  for (int j = J0 + 1; j < J0 + NW; ++j) m = __vmaxu2(m, w[j] & 0x7FFF7FFFu);
  return max(m & 0xFFFFu, m >> 16);
}

// Move the table channel `lw` (0..31) of the block out: return its bits, leave +0 in its slot.
__device__ __forceinline__ uint16_t take_channel(uint32_t (&w)[16], int lw) {
  const int jj = lw >> 1;
  const uint32_t sh = (lw & 1) * 16;
  uint32_t v = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const bool hit = j == jj;
    v |= hit ? w[j] : 0u;
    w[j] &= hit ? ~(0xFFFFu << sh) : 0xFFFFFFFFu;
  }
  return (uint16_t)(v >> sh);
}

// E2M1 codes of 16 consecutive elements (words J0..J0+7) scaled by f, as two u32 (low nibble first).
template <int J0>
__device__ __forceinline__ uint2 codes16(const uint32_t (&w)[16], float f) {
  uint2 r;
  r.x = cvt_e2m1x8(lo_f(w[J0]) * f, hi_f(w[J0]) * f, lo_f(w[J0 + 1]) * f, hi_f(w[J0 + 1]) * f,
                   lo_f(w[J0 + 2]) * f, hi_f(w[J0 + 2]) * f, lo_f(w[J0 + 3]) * f, hi_f(w[J0 + 3]) * f);
  r.y = cvt_e2m1x8(lo_f(w[J0 + 4]) * f, hi_f(w[J0 + 4]) * f, lo_f(w[J0 + 5]) * f, hi_f(w[J0 + 5]) * f,
                   lo_f(w[J0 + 6]) * f, hi_f(w[J0 + 6]) * f, lo_f(w[J0 + 7]) * f, hi_f(w[J0 + 7]) * f);
  return r;
}

// Table facts of one 32-channel block for a thread: up to two table channels (two only for
// G = 16, where the block holds two groups), each with its slot in the block and its B column.
struct BlockTable {
  int lw0, pos0;   // lw < 0: none
  int lw1, pos1;
};

template <int G>
__device__ __forceinline__ BlockTable block_table(int blk, const int8_t* Ls, const int16_t* Ps) {
  BlockTable t{-1, 0, -1, 0};
  if constexpr (G == 32) {
    const int l = Ls[blk];
    if (l >= 0) { t.lw0 = l; t.pos0 = Ps[blk]; }
  } else if constexpr (G == 64) {
    const int g = blk >> 1, l = Ls[g];
    if (l >= 0 && (l >> 5) == (blk & 1)) { t.lw0 = l & 31; t.pos0 = Ps[g]; }
  } else {
    const int l0 = Ls[2 * blk], l1 = Ls[2 * blk + 1];
    if (l0 >= 0) { t.lw0 = l0; t.pos0 = Ps[2 * blk]; }
    if (l1 >= 0) { t.lw1 = 16 + l1; t.pos1 = Ps[2 * blk + 1]; }
  }
  return t;
}

// Stage one table (Kg entries) in shared memory with each entry's B column; returns the
// number of entries (at most K_L). Entries >= G or beyond K_L columns are reported and dropped.
template <int G>
__device__ int stage_table(const int8_t* __restrict__ L, int Kg, int K_L, int8_t* Ls, int16_t* Ps, int* s_warp,
                           int* status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per = (Kg + 255) / 256;
  const int i0 = threadIdx.x * per, i1 = min(Kg, i0 + per);
  int local = 0;
  for (int i = i0; i < i1; ++i) {
    int v = L[i];
    if (v >= G) { record_status(status, DEV_BAD_TABLE); v = -1; }
    Ls[i] = (int8_t)v;
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
  int run = incl - local, count = 0;
  for (int w = 0; w < 8; ++w) { if (w < warp) run += s_warp[w]; count += s_warp[w]; }
  for (int i = i0; i < i1; ++i)
    if (Ls[i] >= 0) {
      if (run >= K_L) { record_status(status, DEV_BAD_TABLE); Ls[i] = -1; }
      Ps[i] = (int16_t)run++;
    }
  __syncthreads();
  return min(count, K_L);
}

// One item = one 32-channel block of one row: extraction, amax, exponent(s), codes, scales.
// All 32 lanes of a warp call it together (the scale words and G = 64 amax use shuffles);
// lanes hold consecutive blocks of the same row (K is a multiple of 256).
template <int G, bool FP8, bool TABLE>
__device__ __forceinline__ void quant_block(uint32_t (&w)[16], int row, int blk, bool live, const BlockTable& t,
                                            int count, int K, int K_L, uint16_t* __restrict__ B,
                                            uint8_t* __restrict__ Q, uint8_t* __restrict__ S) {
  const int lane = threadIdx.x & 31;
  if constexpr (TABLE) {
    if (t.lw0 >= 0) {
      const uint16_t v = take_channel(w, t.lw0);
      if (live) B[(size_t)row * K_L + t.pos0] = v;
    }
    if (G == 16 && t.lw1 >= 0) {
      const uint16_t v = take_channel(w, t.lw1);
      if (live) B[(size_t)row * K_L + t.pos1] = v;
    }
    if (live && blk == 0)
      for (int i = count; i < K_L; ++i) B[(size_t)row * K_L + i] = 0;
  }
  const int nblk = K / 32;
  if constexpr (FP8) {
    const int e = shared_exp<8>(block_amax<0, 16>(w));
    const float f = __uint_as_float((uint32_t)(127 - e) << 23);
    uint32_t c[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      c[j] = cvt_e4m3x4(lo_f(w[2 * j]) * f, hi_f(w[2 * j]) * f, lo_f(w[2 * j + 1]) * f, hi_f(w[2 * j + 1]) * f);
    if (live) {
      uint4* dst = reinterpret_cast<uint4*>(Q + (size_t)row * K + (size_t)blk * 32);
      dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
      dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
    }
    const uint32_t code = (uint32_t)(e + 127);
    const uint32_t c1 = __shfl_down_sync(0xffffffffu, code, 1);
    const uint32_t c2 = __shfl_down_sync(0xffffffffu, code, 2);
    const uint32_t c3 = __shfl_down_sync(0xffffffffu, code, 3);
    if ((blk & 3) == 0)
      *reinterpret_cast<uint32_t*>(S + scale_word_offset(row, blk >> 2, nblk / 4)) = code | (c1 << 8) | (c2 << 16) | (c3 << 24);
  } else if constexpr (G == 16) {
    const int e0 = shared_exp<2>(block_amax<0, 8>(w));
    const int e1 = shared_exp<2>(block_amax<8, 8>(w));
    const uint2 q0 = codes16<0>(w, __uint_as_float((uint32_t)(127 - e0) << 23));
    const uint2 q1 = codes16<8>(w, __uint_as_float((uint32_t)(127 - e1) << 23));
    if (live) *reinterpret_cast<uint4*>(Q + (size_t)row * (K / 2) + (size_t)blk * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    const uint32_t pair = (uint32_t)(e0 + 127) | ((uint32_t)(e1 + 127) << 8);   // slots 2*blk, 2*blk+1
    const uint32_t nxt = __shfl_down_sync(0xffffffffu, pair, 1);
    if ((blk & 1) == 0)
      *reinterpret_cast<uint32_t*>(S + scale_word_offset(row, blk >> 1, nblk / 2)) = pair | (nxt << 16);
  } else {
    uint32_t am = block_amax<0, 16>(w);
    if constexpr (G == 64) am = max(am, __shfl_xor_sync(0xffffffffu, am, 1));
    const int e = shared_exp<2>(am);
    const float f = __uint_as_float((uint32_t)(127 - e) << 23);
    const uint2 q0 = codes16<0>(w, f);
    const uint2 q1 = codes16<8>(w, f);
    if (live) *reinterpret_cast<uint4*>(Q + (size_t)row * (K / 2) + (size_t)blk * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    const uint32_t code = (uint32_t)(e + 127);
    const uint32_t c1 = __shfl_down_sync(0xffffffffu, code, 1);
    const uint32_t c2 = __shfl_down_sync(0xffffffffu, code, 2);
    const uint32_t c3 = __shfl_down_sync(0xffffffffu, code, 3);
    if ((blk & 3) == 0)
      *reinterpret_cast<uint32_t*>(S + scale_word_offset(row, blk >> 2, nblk / 4)) = code | (c1 << 8) | (c2 << 16) | (c3 << 24);
  }
  (void)lane;
}

__device__ __forceinline__ void load_block(const uint16_t* __restrict__ X, size_t off, bool ok, uint32_t (&w)[16]) {
  if (ok) {
    const uint4* p = reinterpret_cast<const uint4*>(X + off);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = __ldg(p + c);
      w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = 0u;
  }
}

constexpr int MAX_KG = 1024;

// Dense form: items (row, 32-channel block) over M rows padded to a multiple of 128 (pad rows
// only get zero scales); each thread takes two items per step so that eight 16-byte loads
// are in flight.
template <int G, bool FP8, bool TABLE>
__global__ void __launch_bounds__(256) quantize_kernel(QuantParams p) {
  __shared__ int8_t s_l[TABLE ? MAX_KG : 1];
  __shared__ int16_t s_pos[TABLE ? MAX_KG : 1];
  __shared__ int s_warp[8];
  const int nblk = p.K / 32;
  const int mpad = (p.M + 127) / 128 * 128;
  const long long items = (long long)mpad * nblk;              // a multiple of 32
  const long long stride = (long long)gridDim.x * 512;
  long long base = (long long)blockIdx.x * 512 + (threadIdx.x & ~31) * 2;
  // the first step's loads go out before the table is staged, so the two latencies overlap
  uint32_t w0[16], w1[16];
  int r0 = 0, b0 = 0, r1 = 0, b1 = 0;
  auto issue = [&](long long b) {
    const long long i0 = b + (threadIdx.x & 31), i1 = i0 + 32;
    r0 = (int)(i0 / nblk); b0 = (int)(i0 - (long long)r0 * nblk);
    r1 = (int)(i1 / nblk); b1 = (int)(i1 - (long long)r1 * nblk);
    load_block(p.X, (size_t)r0 * p.K + (size_t)b0 * 32, b < items && r0 < p.M, w0);
    load_block(p.X, (size_t)r1 * p.K + (size_t)b1 * 32, b + 32 < items && r1 < p.M, w1);
  };
  issue(base);
  int count = 0;
  if constexpr (TABLE) count = stage_table<G>(p.L, p.Kg, p.K_L, s_l, s_pos, s_warp, p.status);
  for (; base < items; base += stride) {
    if (base != (long long)blockIdx.x * 512 + (threadIdx.x & ~31) * 2) issue(base);
    const bool has1 = base + 32 < items;                          // warp-uniform
    BlockTable t0{-1, 0, -1, 0}, t1{-1, 0, -1, 0};
    if constexpr (TABLE) { t0 = block_table<G>(b0, s_l, s_pos); t1 = block_table<G>(b1, s_l, s_pos); }
    quant_block<G, FP8, TABLE>(w0, r0, b0, r0 < p.M, t0, count, p.K, p.K_L, p.B, p.Q, p.S);
    if (has1) quant_block<G, FP8, TABLE>(w1, r1, b1, r1 < p.M, t1, count, p.K, p.K_L, p.B, p.Q, p.S);
  }
}

// Grouped (MoE) form over the padded row space: a row's expert comes from its 128-row block;
// rows past the expert's token count are padding and come out as zeros. The CTA stages every
// expert's table (E x Kg entries) with per-expert B columns.
template <int G>
__global__ void __launch_bounds__(256) quantize_grouped_kernel(GroupedQuantParams p) {
  extern __shared__ __align__(16) unsigned char gsm[];
  const int n = p.E * p.Kg;
  int8_t* s_l = reinterpret_cast<int8_t*>(gsm);
  int16_t* s_pos = reinterpret_cast<int16_t*>(gsm + ((n + 15) & ~15));
  int* s_cnt = reinterpret_cast<int*>(gsm + ((n + 15) & ~15) + ((2 * n + 15) & ~15));
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    int run = 0;
    for (int g = 0; g < p.Kg; ++g) {
      int v = p.L[(size_t)e * p.Kg + g];
      if (v >= G || (v >= 0 && run >= p.K_L)) { record_status(p.status, DEV_BAD_TABLE); v = -1; }
      s_l[e * p.Kg + g] = (int8_t)v;
      if (v >= 0) s_pos[e * p.Kg + g] = (int16_t)run++;
    }
    s_cnt[e] = run;
  }
  __syncthreads();
  const int nblk = p.K / 32;
  const long long items = (long long)p.Mp * nblk;
  for (long long base = (long long)blockIdx.x * 256 + (threadIdx.x & ~31); base < items; base += (long long)gridDim.x * 256) {
    const long long i = base + (threadIdx.x & 31);
    const int row = (int)(i / nblk), blk = (int)(i - (long long)row * nblk);
    const int e = __ldg(p.mblock_expert + row / 128);
    const int local = row - __ldg(p.poff + e);
    const int src0 = __ldg(p.off + e);
    const bool valid = local < __ldg(p.off + e + 1) - src0;
    uint32_t w[16];
    load_block(p.X, (size_t)(src0 + local) * p.K + (size_t)blk * 32, valid, w);
    const BlockTable t = block_table<G>(blk, s_l + e * p.Kg, s_pos + e * p.Kg);
    quant_block<G, false, true>(w, row, blk, true, t, s_cnt[e], p.K, p.K_L, p.B, p.Q, p.S);
  }
}

template <int G, bool FP8, bool TABLE>
static cudaError_t launch_quant(const QuantParams& p, int grid, cudaStream_t s) {
  quantize_kernel<G, FP8, TABLE><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantParams& p, bool fp8, int num_sms, cudaStream_t s) {
  const long long items = (long long)((p.M + 127) / 128 * 128) * (p.K / 32);
  const int grid = (int)std::max<long long>(1, std::min<long long>((items + 511) / 512, (long long)num_sms * 6));
  const bool table = p.L != nullptr;
  if (table && p.Kg > MAX_KG) return cudaErrorInvalidValue;
  if (fp8) return launch_quant<32, true, false>(p, grid, s);
  switch (p.G) {
    case 16: return table ? launch_quant<16, false, true>(p, grid, s) : launch_quant<16, false, false>(p, grid, s);
    case 32: return table ? launch_quant<32, false, true>(p, grid, s) : launch_quant<32, false, false>(p, grid, s);
    case 64: return table ? launch_quant<64, false, true>(p, grid, s) : launch_quant<64, false, false>(p, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

size_t grouped_quant_smem(int E, int Kg) {
  const size_t n = (size_t)E * Kg;
  return ((n + 15) & ~(size_t)15) + ((2 * n + 15) & ~(size_t)15) + (size_t)E * sizeof(int);
}

cudaError_t launch_quantize_grouped(const GroupedQuantParams& p, int num_sms, cudaStream_t s) {
  if (p.Mp == 0) return cudaSuccess;
  const size_t smem = grouped_quant_smem(p.E, p.Kg);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  const long long items = (long long)p.Mp * (p.K / 32);
  const int grid = (int)std::max<long long>(1, std::min<long long>((items + 255) / 256, (long long)num_sms * 4));
  switch (p.G) {
    case 16:
      if (smem > 48 * 1024) cudaFuncSetAttribute(quantize_grouped_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      quantize_grouped_kernel<16><<<grid, 256, smem, s>>>(p); break;
    case 32:
      if (smem > 48 * 1024) cudaFuncSetAttribute(quantize_grouped_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      quantize_grouped_kernel<32><<<grid, 256, smem, s>>>(p); break;
    case 64:
      if (smem > 48 * 1024) cudaFuncSetAttribute(quantize_grouped_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      quantize_grouped_kernel<64><<<grid, 256, smem, s>>>(p); break;
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
