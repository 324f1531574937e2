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

// Byte offset of scale slot `slot` of a row (same layout).
__device__ __forceinline__ size_t scale_byte_offset(int row, int slot, int nslot4) {
  return scale_word_offset(row, slot >> 2, nslot4) + (size_t)(slot & 3);
}

// max(|a|, |b|) per bf16 half; the sign bit of the result is junk (xor of the signs).
__device__ __forceinline__ uint32_t maxabs2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// a * b per bf16 half, round to nearest even. With b a power of two the product is exact
// unless it falls below the normal range (|a * b| < 2^-126); such values are far below the
// first rounding threshold of E2M1 (0.25) and E4M3 (2^-10) and keep their sign, so their
// codes are the same as from the exact product.
__device__ __forceinline__ uint32_t mul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// The bf16 pair (2^-e, 2^-e) for a shared exponent e in [-127, 125].
__device__ __forceinline__ uint32_t pow2_neg_x2(int e) {
  const uint32_t b = (uint32_t)(127 - e) << 7;
  return b | (b << 16);
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

// Largest |x| bits over words [J0, J0+NW) of a 32-element block (bf16 pairs): packed bf16
// max of the magnitudes (finite values order like their bits), then the larger half.
template <int J0, int NW>
__device__ __forceinline__ uint32_t block_amax(const uint32_t (&w)[16]) {
  uint32_t a[NW / 2];
#pragma unroll
  for (int j = 0; j < NW / 2; ++j) a[j] = maxabs2(w[J0 + j], w[J0 + j + NW / 2]);
#pragma unroll
  for (int n = NW / 2; n > 1; n >>= 1)
#pragma unroll
    for (int j = 0; j < n / 2; ++j) a[j] = maxabs2(a[j], a[j + n / 2]);
  const uint32_t m = a[0] & 0x7FFF7FFFu;
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

// E2M1 codes of 16 consecutive elements (words J0..J0+7) scaled by the bf16 pair f2 =
// (2^-e, 2^-e), as two u32 (low nibble first).
template <int J0>
__device__ __forceinline__ uint2 codes16(const uint32_t (&w)[16], uint32_t f2) {
  uint32_t v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = mul2(w[J0 + j], f2);
  uint2 r;
  r.x = cvt_e2m1x8(lo_f(v[0]), hi_f(v[0]), lo_f(v[1]), hi_f(v[1]), lo_f(v[2]), hi_f(v[2]), lo_f(v[3]), hi_f(v[3]));
  r.y = cvt_e2m1x8(lo_f(v[4]), hi_f(v[4]), lo_f(v[5]), hi_f(v[5]), lo_f(v[6]), hi_f(v[6]), lo_f(v[7]), hi_f(v[7]));
  return r;
}

// Table facts of one 32-channel block for a thread: the table entries whose channels fall in
// the block, in table order (group, slot): for G = 32 the R slots of the block's group, for
// G = 16 the R slots of each of its two groups, for G = 64 the slots of its group that lie in
// this half of it. Entry e: the channel within the block (lw, -1 = none) and its B column.
constexpr int BT_SLOTS = 2 * MAX_R;
struct BlockTable {
  int lw[BT_SLOTS];
  int pos[BT_SLOTS];
};

__device__ __forceinline__ BlockTable no_table() {
  BlockTable t;
#pragma unroll
  for (int e = 0; e < BT_SLOTS; ++e) { t.lw[e] = -1; t.pos[e] = 0; }
  return t;
}

// The group holding slot h (h = 0, 1; two only for G = 16) of block blk.
template <int G>
__device__ __forceinline__ int block_group(int blk, int h) {
  return G == 16 ? 2 * blk + h : (G == 64 ? blk >> 1 : blk);
}

// From separate arrays: entry channel (int8) and B column (int16), R slots per group.
template <int G>
__device__ __forceinline__ BlockTable block_table(int blk, const int8_t* Ls, const int16_t* Ps, int R) {
  BlockTable t = no_table();
#pragma unroll
  for (int h = 0; h < (G == 16 ? 2 : 1); ++h)
#pragma unroll
    for (int m = 0; m < MAX_R; ++m) {
      if (m >= R) continue;
      const int i = block_group<G>(blk, h) * R + m;
      const int l = Ls[i];
      if (l < 0 || (G == 64 && (l >> 5) != (blk & 1))) continue;
      t.lw[h * MAX_R + m] = G == 16 ? 16 * h + l : (l & 31);
      t.pos[h * MAX_R + m] = Ps[i];
    }
  return t;
}

// From packed words (column << 8) | (entry & 0xFF), entry -1 (0xFF) meaning none.
template <int G>
__device__ __forceinline__ BlockTable block_table_packed(int blk, const int* tab, int R) {
  BlockTable t = no_table();
#pragma unroll
  for (int h = 0; h < (G == 16 ? 2 : 1); ++h)
#pragma unroll
    for (int m = 0; m < MAX_R; ++m) {
      if (m >= R) continue;
      const int v = tab[block_group<G>(blk, h) * R + m], l = (int)(int8_t)(v & 0xFF);
      if (l < 0 || (G == 64 && (l >> 5) != (blk & 1))) continue;
      t.lw[h * MAX_R + m] = G == 16 ? 16 * h + l : (l & 31);
      t.pos[h * MAX_R + m] = v >> 8;
    }
  return t;
}

// Move the block's table channels out of its 64-byte item in shared memory (64-byte swizzle:
// the 2 bytes of channel lw sit in 16-byte chunk (lw / 8) ^ swz at byte (lw % 8) * 2), in table
// order: each value to its B column of the row (Brow, when live), +0 left in its slot. A
// channel named twice yields its value once and then the 0 the first move left.
template <int G>
__device__ __forceinline__ void extract_from_item(uint8_t* item, int swz, const BlockTable& t, bool loaded, bool live,
                                                  uint16_t* __restrict__ Brow) {
#pragma unroll
  for (int e = 0; e < (G == 16 ? 2 : 1) * MAX_R; ++e) {
    const int lw = t.lw[e];
    if (lw < 0) continue;
    uint16_t* pv = reinterpret_cast<uint16_t*>(item + (((lw >> 3) ^ swz) * 16) + (lw & 7) * 2);
    const uint16_t v = loaded ? *pv : (uint16_t)0;
    if (loaded) *pv = 0;
    if (live) Brow[t.pos[e]] = v;
  }
}

// Stage one table (n = K/G x R entries, in (group, slot) order) in shared memory, packed with
// each entry's B column; returns the number of entries (at most K_L). Entries >= G or beyond
// K_L columns are reported and dropped.
template <int G, int NTHREADS = 256>
__device__ int stage_table(const int8_t* __restrict__ L, int n, int K_L, int* tab, int* s_warp, int* status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per = (n + NTHREADS - 1) / NTHREADS;
  const int i0 = threadIdx.x * per, i1 = min(n, i0 + per);
  int local = 0;
  for (int i = i0; i < i1; ++i) {
    int v = L[i];
    if (v >= G) { record_status(status, DEV_BAD_TABLE); v = -1; }
    tab[i] = v;
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
  for (int w = 0; w < NTHREADS / 32; ++w) { if (w < warp) run += s_warp[w]; count += s_warp[w]; }
  for (int i = i0; i < i1; ++i) {
    const int v = tab[i];
    if (v < 0) { tab[i] = 0xFF; continue; }
    if (run >= K_L) { record_status(status, DEV_BAD_TABLE); tab[i] = 0xFF; }
    else tab[i] = (run << 8) | v;
    ++run;
  }
  __syncthreads();
  return min(count, K_L);
}

// One item = one 32-channel block of one row: extraction, amax, exponent(s), codes, scales.
// All 32 lanes of a warp call it together (for G = 64 the two blocks of a group sit on
// neighbouring lanes and meet by a shuffle); lanes hold consecutive blocks of a row.
// `valid` false: the lane holds no block (a row with fewer blocks than the warp has lanes);
// it still takes part in the G = 64 shuffle but writes nothing.
template <int G, bool FP8, bool TABLE>
__device__ __forceinline__ void quant_block(uint32_t (&w)[16], int row, int blk, bool live, const BlockTable& t,
                                            int count, int K, int K_L, uint16_t* __restrict__ B,
                                            uint8_t* __restrict__ Q, uint8_t* __restrict__ S, bool valid = true) {
  const int lane = threadIdx.x & 31;
  live = live && valid;
  if constexpr (TABLE) {
#pragma unroll
    for (int e = 0; e < (G == 16 ? 2 : 1) * MAX_R; ++e) {
      if (t.lw[e] < 0) continue;
      const uint16_t v = take_channel(w, t.lw[e]);
      if (live) B[(size_t)row * K_L + t.pos[e]] = v;
    }
    if (live && blk == 0)
      for (int i = count; i < K_L; ++i) B[(size_t)row * K_L + i] = 0;
  }
  const int nblk = K / 32;
  if constexpr (FP8) {
    const int e = shared_exp<8>(block_amax<0, 16>(w));
    const uint32_t f2 = pow2_neg_x2(e);
    uint32_t c[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t v0 = mul2(w[2 * j], f2), v1 = mul2(w[2 * j + 1], f2);
      c[j] = cvt_e4m3x4(lo_f(v0), hi_f(v0), lo_f(v1), hi_f(v1));
    }
    if (live) {
      uint4* dst = reinterpret_cast<uint4*>(Q + (size_t)row * K + (size_t)blk * 32);
      dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
      dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
    }
    if (valid) S[scale_byte_offset(row, blk, nblk / 4)] = (uint8_t)(e + 127);
  } else if constexpr (G == 16) {
    const int e0 = shared_exp<2>(block_amax<0, 8>(w));
    const int e1 = shared_exp<2>(block_amax<8, 8>(w));
    const uint2 q0 = codes16<0>(w, pow2_neg_x2(e0));
    const uint2 q1 = codes16<8>(w, pow2_neg_x2(e1));
    if (live) *reinterpret_cast<uint4*>(Q + (size_t)row * (K / 2) + (size_t)blk * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    // slots 2*blk and 2*blk + 1: two neighbouring bytes of one scale word
    if (valid)
      *reinterpret_cast<uint16_t*>(S + scale_byte_offset(row, 2 * blk, nblk / 2)) =
          (uint16_t)((uint32_t)(e0 + 127) | ((uint32_t)(e1 + 127) << 8));
  } else {
    uint32_t am = block_amax<0, 16>(w);
    if constexpr (G == 64) am = max(am, __shfl_xor_sync(0xffffffffu, am, 1));
    const int e = shared_exp<2>(am);
    const uint32_t f2 = pow2_neg_x2(e);
    const uint2 q0 = codes16<0>(w, f2);
    const uint2 q1 = codes16<8>(w, f2);
    if (live) *reinterpret_cast<uint4*>(Q + (size_t)row * (K / 2) + (size_t)blk * 16) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    if (valid) S[scale_byte_offset(row, blk, nblk / 4)] = (uint8_t)(e + 127);
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


// Dense form, TMA-fed. X is viewed as a 2-D tensor of 32-channel blocks (items): rows of 64
// bytes, one per (row, block) in row-major order, so a warp step's 64 items are one
// contiguous 4 KB run of X. Lane 0 loads it with one TMA box in the 64-byte swizzle
// (16-byte chunk c of item r at chunk c ^ ((r / 2) % 4)), which makes every lane's 64-byte
// read from shared memory conflict-free; each warp double-buffers its boxes. Items in rows
// M .. (next multiple of 128) only write zero scales.
constexpr int QSTEP = QUANT_STEP_ITEMS;         // items per warp step (= the TMA box height)
constexpr int QWARPS = 8;
constexpr int QMAXK = 3;                        // CTAs per SM the shared memory allows

__device__ __forceinline__ void load_block_smem(const uint8_t* slot, int r, uint32_t (&w)[16]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(slot + r * 64 + ((c ^ ((r >> 1) & 3)) * 16));
    w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
  }
}

template <int G, bool FP8, bool TABLE>
__global__ void __launch_bounds__(256) quantize_tma_kernel(const __grid_constant__ CUtensorMap tmX, QuantParams p) {
  extern __shared__ uint8_t q_dyn[];      // QWARPS x 2 boxes of 4 KB (1 KB aligned), then the table
  uint8_t* boxes = q_dyn + ((1024u - (smem_u32(q_dyn) & 1023u)) & 1023u);
  auto box_at = [&](int wp, int sl) { return boxes + (wp * 2 + sl) * (QSTEP * 64); };
  int* s_tab = reinterpret_cast<int*>(boxes + QWARPS * 2 * QSTEP * 64);   // K/G x R packed entries
  __shared__ __align__(8) uint64_t s_bar[QWARPS][2];
  __shared__ int s_warp[8];
  __shared__ int s_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nblk = p.K / 32;
  const uint32_t mpad = (uint32_t)(p.M + 127) / 128 * 128;
  const uint32_t items = mpad * (uint32_t)nblk;             // a multiple of 64
  const uint32_t real_items = (uint32_t)p.M * (uint32_t)nblk;
  const uint32_t nsteps = items / QSTEP;
  // CTA b takes a contiguous run of nsteps / grid steps (one more for the first nsteps % grid
  // CTAs), so the left-over steps fall on different SMs and a CTA's loads cover one stretch of
  // X; its warps take the run's steps round robin
  const uint32_t wstride = QWARPS;
  const uint32_t per = nsteps / gridDim.x, extra = nsteps % gridDim.x;
  const uint32_t cta_first = blockIdx.x * per + min(blockIdx.x, extra);
  const uint32_t cta_end = cta_first + per + (blockIdx.x < extra ? 1u : 0u);
  uint32_t step = cta_first + warp;
  if (threadIdx.x == 0) s_abort = 0;
  if (lane == 0) { mbar_init(smem_u32(&s_bar[warp][0]), 1); mbar_init(smem_u32(&s_bar[warp][1]), 1); }
  fence_barrier_init();
  __syncwarp();
  // X, L and the outputs are free of the previous kernel. The next kernel (normally the
  // product, whose CTAs need a whole SM) may launch at once: its CTAs take the SMs this grid's
  // CTAs leave and run their prologue while the rest of this grid finishes (QKV step 36.9 ->
  // 36.4 us). A next grid of this kernel would instead hold SM slots while it waits (a graph
  // of quantize launches alone: 7.7 -> 8.5 us per launch).
  grid_dep_wait();
  if (threadIdx.x == 0) grid_dep_launch();
  // both of the warp's first boxes go out before the table is staged, so the whole first
  // wave of loads is in flight while the table comes in
  auto issue = [&](uint32_t st, int slot) {
    if (lane == 0 && st * QSTEP < real_items) {
      const uint32_t bar = smem_u32(&s_bar[warp][slot]);
      mbar_arrive_expect_tx(bar, QSTEP * 64);
      tma_load_2d(smem_u32(box_at(warp, slot)), &tmX, 0, (int)(st * QSTEP), bar);
    }
  };
  if (step < cta_end) issue(step, 0);
  if (step + wstride < cta_end) issue(step + wstride, 1);
  int count = 0;
  if constexpr (TABLE) count = stage_table<G>(p.L, p.Kg * p.R, p.K_L, s_tab, s_warp, p.status);
  else __syncthreads();
  uint32_t phbits = 0;                                        // bit s: parity of slot s's next phase
  int slot = 0;
  for (; step < cta_end; step += wstride, slot ^= 1) {
    const bool loaded = step * QSTEP < real_items;            // warp-uniform (pad rows are not loaded)
    if (loaded) {
      // lane 0 waits (bounded) and the warp follows its result; __syncwarp then orders the
      // other lanes' shared-memory reads after the completed load
      bool ok = true;
      if (lane == 0) ok = mbar_wait(smem_u32(&s_bar[warp][slot]), (phbits >> slot) & 1u, reinterpret_cast<volatile int*>(&s_abort), p.status);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      __syncwarp();
      if (!ok) {
        // let the other slot's load (if one was issued) land before leaving
        if (lane == 0 && step + wstride < cta_end && (step + wstride) * QSTEP < real_items) {
          volatile int never = 0;
          mbar_wait(smem_u32(&s_bar[warp][slot ^ 1]), (phbits >> (slot ^ 1)) & 1u, &never, nullptr, 100000000ull);
        }
        break;
      }
      phbits ^= 1u << slot;
    }
    uint8_t* box = box_at(warp, slot);
    // rows and blocks of this lane's two items (one division per step, then carries)
    const uint32_t it0 = step * QSTEP;
    int rowa = (int)(it0 / (uint32_t)nblk);
    int blka = (int)(it0 - (uint32_t)rowa * nblk) + lane;
    while (blka >= nblk) { blka -= nblk; ++rowa; }
    // the lane's items in three passes (extraction, loads, quantization), so that the
    // quantization of its items is independent work the scheduler can interleave (QKV quantize
    // 8.52 -> 8.39 us against one item after the other)
    constexpr int NH = QSTEP / 32;
    int rows[NH], blks[NH];
    bool lives[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const int r = lane + 32 * h;                            // item within the box
      int row = rowa, blk = blka + 32 * h;
      while (blk >= nblk) { blk -= nblk; ++row; }
      rows[h] = row; blks[h] = blk; lives[h] = row < p.M;
      if constexpr (TABLE) {
        // move the table channels out of the box (in table order), then clear B's pad columns
        const BlockTable t = block_table_packed<G>(blk, s_tab, p.R);
        extract_from_item<G>(box + r * 64, (r >> 1) & 3, t, loaded, lives[h], p.B + (size_t)row * p.K_L);
        if (lives[h] && blk == 0)
          for (int i = count; i < p.K_L; ++i) p.B[(size_t)row * p.K_L + i] = 0;
      }
    }
    uint32_t w[NH][16];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      if (loaded) load_block_smem(box, lane + 32 * h, w[h]);  // rows past M arrive zero-filled
      else {
#pragma unroll
        for (int j = 0; j < 16; ++j) w[h][j] = 0u;
      }
    }
#pragma unroll
    for (int h = 0; h < NH; ++h)
      quant_block<G, FP8, false>(w[h], rows[h], blks[h], lives[h], no_table(), count, p.K, p.K_L, p.B, p.Q, p.S);
    __syncwarp();                                             // every lane is done with this slot
    if (step + 2 * wstride < cta_end) { fence_proxy_async_smem(); issue(step + 2 * wstride, slot); }
  }
}

// Producer-fused form: RMSNorm of each row, then extraction and MX quantization of the
// normalized row, in one pass over X (Figure 2 of the OSC page puts extraction and
// microscaling right before the GEMM; the RMSNorm that produces the projection's input is
// the step before them). A warp owns a row: the row's sum of squares must be complete before
// any block can be scaled. Rows arrive by one TMA box each ({32 channels, K/32 blocks}, the
// 64-byte swizzle of the dense kernel) into a per-warp double buffer; gamma is staged once per
// CTA in the same swizzle. Arithmetic, every step rounded to nearest even in fp32 with no
// fused multiply-add: s_b = x_0^2 + ... + x_31^2 per 32-channel block in ascending order; the
// block sums, padded with zeros to a power of two, combined pairwise (s_b += s_{b+h} for
// h = P/2 .. 1); inv = 1 / sqrt(total / K + eps); y = bf16((x * inv) * gamma).
constexpr int NQ_WARPS = 16;
constexpr int NQ_THREADS = NQ_WARPS * 32;
constexpr int NQ_PARTS = 8;                      // block sums per lane: a power of two >= NQ_MAX_K / 1024
static_assert(NQ_PARTS * 1024 >= NQ_MAX_K && (NQ_PARTS & (NQ_PARTS - 1)) == 0, "block sums per lane");

// Row buffers per warp: two (the next row loads while this one is computed) when they fit in
// shared memory beside gamma, else one.
__host__ __device__ constexpr int nq_slots(int K) {
  return (size_t)(((size_t)K * 2 + 1023) & ~(size_t)1023) * (1 + 2 * NQ_WARPS) + 1024 <= 227 * 1024 ? 2 : 1;
}

template <int G, bool TABLE>
__global__ void __launch_bounds__(NQ_THREADS, 1) rmsnorm_quantize_kernel(const __grid_constant__ CUtensorMap tmX, NormQuantParams p) {
  extern __shared__ uint8_t nq_dyn[];
  uint8_t* base = nq_dyn + ((1024u - (smem_u32(nq_dyn) & 1023u)) & 1023u);
  const int nb = p.K / 32;                                   // 32-channel blocks per row
  const int nslots = nq_slots(p.K);
  const uint32_t row_bytes = (uint32_t)p.K * 2u;
  const uint32_t slot_bytes = (row_bytes + 1023u) & ~1023u;
  uint8_t* gam = base;
  auto row_buf = [&](int wp, int sl) { return base + slot_bytes * (1u + (uint32_t)(wp * nslots + sl)); };
  __shared__ __align__(8) uint64_t s_bar[NQ_WARPS][2];
  __shared__ __align__(8) int s_tab[TABLE ? NQ_MAX_K / 16 * MAX_R : 2];
  __shared__ int s_warp[NQ_WARPS];
  __shared__ int s_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t mpad = (uint32_t)(p.M + 127) / 128u * 128u;
  // CTA b takes a contiguous run of rows (one more for the first mpad % grid CTAs); its warps
  // take the run's rows round robin; the warp's j-th row uses buffer j % nslots
  const uint32_t per = mpad / gridDim.x, extra = mpad % gridDim.x;
  const uint32_t first = blockIdx.x * per + min(blockIdx.x, extra);
  const uint32_t end = first + per + (blockIdx.x < extra ? 1u : 0u);
  if (threadIdx.x == 0) s_abort = 0;
  if (lane == 0) { mbar_init(smem_u32(&s_bar[warp][0]), 1); mbar_init(smem_u32(&s_bar[warp][1]), 1); }
  fence_barrier_init();
  __syncwarp();
  grid_dep_wait();                                           // X, gamma and L are free of the previous kernel
  if (threadIdx.x == 0) grid_dep_launch();                   // the product may launch now (see the dense kernel)
  auto issue = [&](uint32_t r, int slot) {
    if (lane == 0 && r < end && r < (uint32_t)p.M) {
      const uint32_t bar = smem_u32(&s_bar[warp][slot]);
      mbar_arrive_expect_tx(bar, row_bytes);
      tma_load_2d(smem_u32(row_buf(warp, slot)), &tmX, 0, (int)(r * (uint32_t)nb), bar);
    }
  };
  const uint32_t row0 = first + warp;
  for (int sl = 0; sl < nslots; ++sl) issue(row0 + (uint32_t)sl * NQ_WARPS, sl);
  for (int i = threadIdx.x; i < nb * 4; i += blockDim.x) {  // gamma, 16-byte chunks, swizzled
    const int b = i >> 2, c = i & 3;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.gamma) + i);
    *reinterpret_cast<uint4*>(gam + b * 64 + ((c ^ ((b >> 1) & 3)) * 16)) = v;
  }
  int count = 0;
  if constexpr (TABLE) count = stage_table<G, NQ_THREADS>(p.L, p.Kg * p.R, p.K_L, s_tab, s_warp, p.status);
  else __syncthreads();
  const int iters = (nb + 31) / 32;                          // blocks per lane (<= NQ_PARTS)
  uint32_t phbits = 0;
  int slot = 0;
  for (uint32_t row = row0; row < end; row += NQ_WARPS, slot = (slot + 1 == nslots) ? 0 : slot + 1) {
    const bool loaded = row < (uint32_t)p.M;                 // warp-uniform (pad rows are not loaded)
    if (loaded) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(smem_u32(&s_bar[warp][slot]), (phbits >> slot) & 1u, reinterpret_cast<volatile int*>(&s_abort), p.status);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      __syncwarp();
      if (!ok) {
        // let the other buffer's load (if one was issued) land before leaving
        const uint32_t nxt = row + NQ_WARPS;
        if (lane == 0 && nslots == 2 && nxt < end && nxt < (uint32_t)p.M) {
          const int o = slot ^ 1;
          volatile int never = 0;
          mbar_wait(smem_u32(&s_bar[warp][o]), (phbits >> o) & 1u, &never, nullptr, 100000000ull);
        }
        break;
      }
      phbits ^= 1u << slot;
    }
    const uint8_t* buf = row_buf(warp, slot);
    float inv = 0.0f;
    if (loaded) {
      float part[NQ_PARTS];
#pragma unroll
      for (int i = 0; i < NQ_PARTS; ++i) {
        part[i] = 0.0f;
        const int blk = lane + 32 * i;
        if (i < iters && blk < nb) {
          uint32_t w[16];
          load_block_smem(buf, blk, w);
          float acc = 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float lo = lo_f(w[j]), hi = hi_f(w[j]);
            acc = __fadd_rn(acc, __fmul_rn(lo, lo));
            acc = __fadd_rn(acc, __fmul_rn(hi, hi));
          }
          part[i] = acc;
        }
      }
      // pairwise over the blocks: first the levels whose partners sit in the same lane
      // (h = 32 hh blocks apart), then across lanes; levels above the row's own power of two
      // only add zeros, which changes nothing
#pragma unroll
      for (int hh = NQ_PARTS / 2; hh >= 1; hh >>= 1)
#pragma unroll
        for (int i = 0; i < hh; ++i) part[i] = __fadd_rn(part[i], part[i + hh]);
      float v = part[0];
#pragma unroll
      for (int h = 16; h >= 1; h >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, h));
      const float total = __shfl_sync(0xffffffffu, v, 0);
      const float root = __fsqrt_rn(__fadd_rn(__fdiv_rn(total, (float)p.K), p.eps));
      inv = __fdiv_rn(1.0f, root);
    }
    for (int i = 0; i < iters; ++i) {
      const int blk = lane + 32 * i;
      const bool valid = blk < nb;
      const bool here = loaded && valid;                      // the lane holds a block of a real row
      // the normalized block goes back over its x in the row buffer (same swizzle), so the
      // table channels move out by address, as in the dense kernel, rather than by a select
      // over the block's registers (fused quantize 11.85 -> 11.2 us at QKV M = 2048)
      uint8_t* item = const_cast<uint8_t*>(buf) + blk * 64;
      const int swz = (blk >> 1) & 3;
      uint32_t w[16];
      if (here) {
        uint32_t x[16], g[16];
        load_block_smem(buf, blk, x);
        load_block_smem(gam, blk, g);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float ylo = __fmul_rn(__fmul_rn(lo_f(x[j]), inv), lo_f(g[j]));
          const float yhi = __fmul_rn(__fmul_rn(hi_f(x[j]), inv), hi_f(g[j]));
          w[j] = pack_bf16x2(ylo, yhi);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(item + ((c ^ swz) * 16)) = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      }
      if constexpr (TABLE) {
        if (valid) {
          const BlockTable t = block_table_packed<G>(blk, s_tab, p.R);
          extract_from_item<G>(item, swz, t, here, here, p.B + (size_t)row * p.K_L);
        }
        if (loaded && blk == 0)                               // B's pad columns of a real row
          for (int c = count; c < p.K_L; ++c) p.B[(size_t)row * p.K_L + c] = 0;
      }
      if (here) load_block_smem(buf, blk, w);
      else {
#pragma unroll
        for (int j = 0; j < 16; ++j) w[j] = 0u;
      }
      quant_block<G, false, false>(w, (int)row, blk, loaded, no_table(), count, p.K, p.K_L, p.B, p.Q, p.S, valid);
    }
    __syncwarp();                                             // every lane is done with this buffer
    const uint32_t nxt = row + (uint32_t)nslots * NQ_WARPS;
    if (nxt < end) { fence_proxy_async_smem(); issue(nxt, slot); }
  }
}

size_t rmsnorm_quant_smem(int K) {
  const size_t slot = ((size_t)K * 2 + 1023) & ~(size_t)1023;
  return slot * (1 + (size_t)nq_slots(K) * NQ_WARPS) + 1024;
}

template <int G, bool TABLE>
static cudaError_t launch_nq(const CUtensorMap& tmX, const NormQuantParams& p, int grid, size_t smem, cudaStream_t s) {
  static PerDeviceOnce smem_attr;
  const cudaError_t ae = smem_attr.run([] {
    return cudaFuncSetAttribute(rmsnorm_quantize_kernel<G, TABLE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)rmsnorm_quant_smem(NQ_MAX_K));   // the largest K needs the most
  });
  if (ae != cudaSuccess) return ae;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(NQ_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, rmsnorm_quantize_kernel<G, TABLE>, tmX, p);
}

cudaError_t launch_rmsnorm_quantize(const CUtensorMap& tmX, const NormQuantParams& p, int num_sms, cudaStream_t s) {
  if (p.K % 256 != 0 || p.K > NQ_MAX_K) return cudaErrorInvalidValue;
  const bool table = p.L != nullptr;
  if (table && p.Kg * p.R > NQ_MAX_K / 16 * MAX_R) return cudaErrorInvalidValue;
  const size_t smem = rmsnorm_quant_smem(p.K);
  const long long rows = (long long)(p.M + 127) / 128 * 128;
  // one CTA of 16 warps per SM (its registers, up to 128 a thread, fill the SM's file)
  const int grid = (int)std::max<long long>(1, std::min<long long>((rows + NQ_WARPS - 1) / NQ_WARPS, (long long)num_sms));
  switch (p.G) {
    case 16: return table ? launch_nq<16, true>(tmX, p, grid, smem, s) : launch_nq<16, false>(tmX, p, grid, smem, s);
    case 32: return table ? launch_nq<32, true>(tmX, p, grid, smem, s) : launch_nq<32, false>(tmX, p, grid, smem, s);
    case 64: return table ? launch_nq<64, true>(tmX, p, grid, smem, s) : launch_nq<64, false>(tmX, p, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

// Grouped (MoE) form on the TMA design of the dense kernel. The T routed rows of X are dense
// and sorted by expert; steps of QSTEP items run over them exactly as in the dense kernel, and
// each item's output row is its row in the padded space, poff[e] + t - off[e] for the expert
// e that owns dense row t. The padded space's other rows take zero codes, scales and B in a
// tail phase: pad row p (0 <= p < Mp - T) belongs to the expert e with
// poff[e] - off[e] <= p < poff[e+1] - off[e+1] and sits at row off[e+1] + p.
// Shared memory after the boxes: every expert's packed table (E x Kg words), off, poff (E+1
// each) and the experts' entry counts (E).
__device__ __forceinline__ int last_le(const int* a, int n, int v) {   // largest i < n with a[i] <= v (a[0] <= v)
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

size_t grouped_tma_smem(int E, int Kg, int R) {
  return (size_t)QWARPS * 2 * QSTEP * 64 + 1024 + 4 * ((size_t)E * Kg * R + 2 * ((size_t)E + 1) + (size_t)E);
}

template <int G>
__global__ void __launch_bounds__(256) quantize_grouped_tma_kernel(const __grid_constant__ CUtensorMap tmX,
                                                                    GroupedQuantParams p, int T) {
  extern __shared__ uint8_t q_dyn[];
  uint8_t* boxes = q_dyn + ((1024u - (smem_u32(q_dyn) & 1023u)) & 1023u);
  auto box_at = [&](int wp, int sl) { return boxes + (wp * 2 + sl) * (QSTEP * 64); };
  const int nt = p.Kg * p.R;                                 // table entries per expert
  int* s_tab = reinterpret_cast<int*>(boxes + QWARPS * 2 * QSTEP * 64);
  int* s_off = s_tab + p.E * nt;
  int* s_poff = s_off + (p.E + 1);
  int* s_cnt = s_poff + (p.E + 1);
  __shared__ __align__(8) uint64_t s_bar[QWARPS][2];
  __shared__ int s_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nblk = p.K / 32;
  const uint32_t real_items = (uint32_t)T * (uint32_t)nblk;
  const uint32_t nsteps = (real_items + QSTEP - 1) / QSTEP;
  const uint32_t wstride = QWARPS;
  const uint32_t per = nsteps / gridDim.x, extra = nsteps % gridDim.x;
  const uint32_t cta_first = blockIdx.x * per + min(blockIdx.x, extra);
  const uint32_t cta_end = cta_first + per + (blockIdx.x < extra ? 1u : 0u);
  uint32_t step = cta_first + warp;
  if (threadIdx.x == 0) s_abort = 0;
  if (lane == 0) { mbar_init(smem_u32(&s_bar[warp][0]), 1); mbar_init(smem_u32(&s_bar[warp][1]), 1); }
  fence_barrier_init();
  __syncwarp();
  grid_dep_wait();
  if (threadIdx.x == 0) grid_dep_launch();                   // the product may launch now (see the dense kernel)
  auto issue = [&](uint32_t st, int slot) {
    if (lane == 0) {
      const uint32_t bar = smem_u32(&s_bar[warp][slot]);
      mbar_arrive_expect_tx(bar, QSTEP * 64);                  // a box past the last item is zero-filled
      tma_load_2d(smem_u32(box_at(warp, slot)), &tmX, 0, (int)(st * QSTEP), bar);
    }
  };
  if (step < cta_end) issue(step, 0);
  if (step + wstride < cta_end) issue(step + wstride, 1);
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) { s_off[i] = p.off[i]; s_poff[i] = p.poff[i]; }
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {     // one thread per expert table
    int run = 0;
    for (int g = 0; g < nt; ++g) {
      int v = p.L[(size_t)e * nt + g];
      if (v >= G || (v >= 0 && run >= p.K_L)) { record_status(p.status, DEV_BAD_TABLE); v = -1; }
      s_tab[e * nt + g] = v < 0 ? 0xFF : ((run++ << 8) | v);
    }
    s_cnt[e] = run;
  }
  __syncthreads();
  uint32_t phbits = 0;
  int slot = 0;
  for (; step < cta_end; step += wstride, slot ^= 1) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(smem_u32(&s_bar[warp][slot]), (phbits >> slot) & 1u, reinterpret_cast<volatile int*>(&s_abort), p.status);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    if (!ok) {
      if (lane == 0 && step + wstride < cta_end) {
        volatile int never = 0;
        mbar_wait(smem_u32(&s_bar[warp][slot ^ 1]), (phbits >> (slot ^ 1)) & 1u, &never, nullptr, 100000000ull);
      }
      break;
    }
    phbits ^= 1u << slot;
    uint8_t* box = box_at(warp, slot);
    const uint32_t it0 = step * QSTEP;
    int ta = (int)(it0 / (uint32_t)nblk);                     // dense row and block of item `lane`
    int blka = (int)(it0 - (uint32_t)ta * nblk) + lane;
    while (blka >= nblk) { blka -= nblk; ++ta; }
    int e_row = -1, e = 0, dest0 = 0;                         // expert lookup cached per dense row
    // three passes over the lane's items (extraction, loads, quantization), as in the dense kernel
    constexpr int NH = QSTEP / 32;
    int rows[NH], blks[NH];
    bool lives[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const int r = lane + 32 * h;
      int t = ta, blk = blka + 32 * h;
      while (blk >= nblk) { blk -= nblk; ++t; }
      const bool live = t < T;
      if (live && t != e_row) {
        e = last_le(s_off, p.E + 1, t);                       // the non-empty expert holding row t
        dest0 = s_poff[e] - s_off[e];
        e_row = t;
      }
      const int row = live ? dest0 + t : 0;
      rows[h] = row; blks[h] = blk; lives[h] = live;
      const BlockTable tb = live ? block_table_packed<G>(blk, s_tab + e * nt, p.R) : no_table();
      extract_from_item<G>(box + r * 64, (r >> 1) & 3, tb, true, live, p.B + (size_t)row * p.K_L);
      if (live && blk == 0)
        for (int i = s_cnt[e]; i < p.K_L; ++i) p.B[(size_t)row * p.K_L + i] = 0;
    }
    uint32_t w[NH][16];
#pragma unroll
    for (int h = 0; h < NH; ++h) load_block_smem(box, lane + 32 * h, w[h]);
#pragma unroll
    for (int h = 0; h < NH; ++h)
      quant_block<G, false, false>(w[h], rows[h], blks[h], lives[h], no_table(), 0, p.K, p.K_L, p.B, p.Q, p.S,
                                   lives[h]);
    __syncwarp();
    if (step + 2 * wstride < cta_end) { fence_proxy_async_smem(); issue(step + 2 * wstride, slot); }
  }
  // tail: the padded space's rows past each expert's tokens get zero codes, scales and B
  const uint32_t pad_items = (uint32_t)(p.Mp - T) * (uint32_t)nblk;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < pad_items; i += gridDim.x * blockDim.x) {
    const int pr = (int)(i / (uint32_t)nblk), blk = (int)(i - (uint32_t)pr * nblk);
    int lo = 0, hi = p.E - 1;                                 // largest e with poff[e] - off[e] <= pr
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_poff[mid] - s_off[mid] <= pr) lo = mid; else hi = mid - 1;
    }
    const int row = s_off[lo + 1] + pr;
    *reinterpret_cast<uint4*>(p.Q + (size_t)row * (p.K / 2) + (size_t)blk * 16) = make_uint4(0u, 0u, 0u, 0u);
    if (G == 16) *reinterpret_cast<uint16_t*>(p.S + scale_byte_offset(row, 2 * blk, nblk / 2)) = 0;
    else p.S[scale_byte_offset(row, blk, nblk / 4)] = 0;
    if (blk == 0)
      for (int c = 0; c < p.K_L; ++c) p.B[(size_t)row * p.K_L + c] = 0;
  }
}

template <int G>
static cudaError_t launch_grouped_tma_g(const CUtensorMap& tmX, const GroupedQuantParams& p, int T, int grid,
                                        size_t smem, cudaStream_t s) {
  static PerDeviceOnce smem_attr;
  const cudaError_t ae = smem_attr.run([] {
    return cudaFuncSetAttribute(quantize_grouped_tma_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GROUPED_TMA_SMEM_MAX);
  });
  if (ae != cudaSuccess) return ae;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_grouped_tma_kernel<G>, tmX, p, T);
}

// T = off[E], the routed rows of X (the tensor map covers exactly these rows).
cudaError_t launch_quantize_grouped_tma(const CUtensorMap& tmX, const GroupedQuantParams& p, int T, int num_sms,
                                        cudaStream_t s) {
  if (p.Mp == 0) return cudaSuccess;
  const size_t smem = grouped_tma_smem(p.E, p.Kg, p.R);
  if (smem > (size_t)GROUPED_TMA_SMEM_MAX) return cudaErrorInvalidValue;
  const int per_sm = std::max(1, std::min(QMAXK, (int)(227 * 1024 / (smem + 1024))));
  const long long steps = std::max<long long>(1, ((long long)T * (p.K / 32) + QSTEP - 1) / QSTEP);
  int grid = 1;
  long long best = -1;
  for (int k = 1; k <= per_sm; ++k) {
    const long long ctas = std::max<long long>(1, std::min<long long>((steps + QWARPS - 1) / QWARPS, (long long)num_sms * k));
    const long long busiest = ((steps + ctas - 1) / ctas + QWARPS - 1) / QWARPS;
    if (best < 0 || busiest <= best) { best = busiest; grid = (int)ctas; }
  }
  switch (p.G) {
    case 16: return launch_grouped_tma_g<16>(tmX, p, T, grid, smem, s);
    case 32: return launch_grouped_tma_g<32>(tmX, p, T, grid, smem, s);
    case 64: return launch_grouped_tma_g<64>(tmX, p, T, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

// Grouped (MoE) form, one lane per block with plain loads: the fallback for tables too large
// to stage beside the TMA boxes. Over the padded row space: a row's expert comes from its 128-row block;
// rows past the expert's token count are padding and come out as zeros. The CTA stages every
// expert's table (E x K/G x R entries) with per-expert B columns.
template <int G>
__global__ void __launch_bounds__(256) quantize_grouped_kernel(GroupedQuantParams p) {
  extern __shared__ __align__(16) unsigned char gsm[];
  const int nt = p.Kg * p.R;                                 // table entries per expert
  const int n = p.E * nt;
  int8_t* s_l = reinterpret_cast<int8_t*>(gsm);
  int16_t* s_pos = reinterpret_cast<int16_t*>(gsm + ((n + 15) & ~15));
  int* s_cnt = reinterpret_cast<int*>(gsm + ((n + 15) & ~15) + ((2 * n + 15) & ~15));
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    int run = 0;
    for (int g = 0; g < nt; ++g) {
      int v = p.L[(size_t)e * nt + g];
      if (v >= G || (v >= 0 && run >= p.K_L)) { record_status(p.status, DEV_BAD_TABLE); v = -1; }
      s_l[e * nt + g] = (int8_t)v;
      if (v >= 0) s_pos[e * nt + g] = (int16_t)run++;
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
    const BlockTable t = block_table<G>(blk, s_l + e * nt, s_pos + e * nt, p.R);
    quant_block<G, false, true>(w, row, blk, true, t, s_cnt[e], p.K, p.K_L, p.B, p.Q, p.S);
  }
}

constexpr int QSMEM = QWARPS * 2 * QSTEP * 64 + 1024;

// Dynamic shared memory of the dense kernel: the boxes, then the table (n entries).
size_t quant_smem(int n_table) { return (size_t)QSMEM + (((size_t)n_table * 4 + 15) & ~(size_t)15); }

template <int G, bool FP8, bool TABLE>
static cudaError_t launch_quant(const CUtensorMap& tmX, const QuantParams& p, int grid, size_t smem, cudaStream_t s) {
  static PerDeviceOnce smem_attr;
  const cudaError_t ae = smem_attr.run([] {
    return cudaFuncSetAttribute(quantize_tma_kernel<G, FP8, TABLE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)quant_smem(MAX_TAB));
  });
  if (ae != cudaSuccess) return ae;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_tma_kernel<G, FP8, TABLE>, tmX, p);
}

cudaError_t launch_quantize(const CUtensorMap& tmX, const QuantParams& p, bool fp8, int num_sms, cudaStream_t s) {
  // 1..3 CTAs per SM: the fewest steps for the busiest warp (the critical path; a CTA's run of
  // ceil(steps / CTAs) steps is shared by its QWARPS warps), and on a tie the most resident warps
  // (more warps per scheduler hide more of each warp's latency)
  const bool table = p.L != nullptr;
  const int n_table = table ? p.Kg * p.R : 0;
  if (n_table > MAX_TAB) return cudaErrorInvalidValue;
  const size_t smem = quant_smem(n_table);
  // resident CTAs per SM: at most QMAXK, fewer when a large table grows the shared memory
  // (each CTA also holds ~1 KB of static and system shared memory)
  const int fit = (int)std::max<size_t>(1, (size_t)232448 / (smem + 2048));
  const long long steps = (long long)((p.M + 127) / 128 * 128) * (p.K / 32) / QSTEP;
  int grid = 1;
  long long best = -1;
  for (int k = 1; k <= std::min(QMAXK, fit); ++k) {
    const long long ctas = std::max<long long>(1, std::min<long long>((steps + QWARPS - 1) / QWARPS, (long long)num_sms * k));
    const long long busiest = ((steps + ctas - 1) / ctas + QWARPS - 1) / QWARPS;
    if (best < 0 || busiest <= best) { best = busiest; grid = (int)ctas; }
  }
  if (fp8) return launch_quant<32, true, false>(tmX, p, grid, smem, s);
  switch (p.G) {
    case 16: return table ? launch_quant<16, false, true>(tmX, p, grid, smem, s) : launch_quant<16, false, false>(tmX, p, grid, smem, s);
    case 32: return table ? launch_quant<32, false, true>(tmX, p, grid, smem, s) : launch_quant<32, false, false>(tmX, p, grid, smem, s);
    case 64: return table ? launch_quant<64, false, true>(tmX, p, grid, smem, s) : launch_quant<64, false, false>(tmX, p, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

size_t grouped_quant_smem(int E, int Kg, int R) {
  const size_t n = (size_t)E * Kg * R;
  return ((n + 15) & ~(size_t)15) + ((2 * n + 15) & ~(size_t)15) + (size_t)E * sizeof(int);
}

cudaError_t launch_quantize_grouped(const GroupedQuantParams& p, int num_sms, cudaStream_t s) {
  if (p.Mp == 0) return cudaSuccess;
  const size_t smem = grouped_quant_smem(p.E, p.Kg, p.R);
  if (smem > GROUPED_QUANT_SMEM_MAX) return cudaErrorInvalidValue;
  const long long items = (long long)p.Mp * (p.K / 32);
  const int grid = (int)std::max<long long>(1, std::min<long long>((items + 255) / 256, (long long)num_sms * 4));
  // the attribute is raised once per device to the largest table size the entry point accepts,
  // so no later call with more experts needs a new setting
  static PerDeviceOnce attr[3];
  auto raise = [](auto kern) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GROUPED_QUANT_SMEM_MAX);
  };
  cudaError_t e;
  switch (p.G) {
    case 16:
      if ((e = attr[0].run([&] { return raise(quantize_grouped_kernel<16>); })) != cudaSuccess) return e;
      quantize_grouped_kernel<16><<<grid, 256, smem, s>>>(p); break;
    case 32:
      if ((e = attr[1].run([&] { return raise(quantize_grouped_kernel<32>); })) != cudaSuccess) return e;
      quantize_grouped_kernel<32><<<grid, 256, smem, s>>>(p); break;
    case 64:
      if ((e = attr[2].run([&] { return raise(quantize_grouped_kernel<64>); })) != cudaSuccess) return e;
      quantize_grouped_kernel<64><<<grid, 256, smem, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// W_L (§3.2/§3.3): the bf16 weight columns of the table's channels, one contiguous
// N x K_L block in table order (group, slot); pad columns are zero.
__global__ void __launch_bounds__(256) gather_wl_kernel(const uint16_t* __restrict__ W, int N, int K, int G,
                                                        const int8_t* __restrict__ L, int n_table, int R, int K_L,
                                                        uint16_t* __restrict__ WL, int* status) {
  extern __shared__ int chan[];          // K_L entries: source channel, or -1 for pad
  if (threadIdx.x == 0) {
    int c = 0;
    for (int i = 0; i < n_table; ++i) {
      const int v = L[i];
      if (v >= G) { record_status(status, DEV_BAD_TABLE); continue; }
      if (v < 0) continue;
      if (c >= K_L) { record_status(status, DEV_BAD_TABLE); break; }
      chan[c++] = (i / R) * G + v;
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

cudaError_t launch_gather_wl(const uint16_t* W, int N, int K, int G, const int8_t* L, int R, int K_L, uint16_t* WL,
                             int* status, int num_sms, cudaStream_t s) {
  if (K_L == 0 || N == 0) return cudaSuccess;
  long long total = (long long)N * K_L;
  int grid = (int)std::min<long long>((total + 255) / 256, (long long)num_sms * 4);
  gather_wl_kernel<<<grid, 256, (size_t)K_L * sizeof(int), s>>>(W, N, K, G, L, (K / G) * R, R, K_L, WL, status);
  return cudaGetLastError();
}

}  // namespace osc
