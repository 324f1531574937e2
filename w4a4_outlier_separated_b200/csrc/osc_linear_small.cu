// Split-K OSC dual-path linear for few token rows (M <= 16), the weight-bound regime of
// decoding:
//
//   Y = (Q_X (x) Q_W) * S  +  B * W_L          (the OSC page, §3.2)
//
// computed transposed, Y^T = Q_W (x) Q_X^T + W_L * B^T: the weight tile is the MMA's 128-row
// operand and the token rows its N = 16, so the tensor-core work scales with the real token
// count instead of a 128-row tile that is mostly padding (a 128 x 16 block-scaled MMA costs an
// eighth of a 128 x 128 one). What remains is streaming the weights: Q_W, S_W and W_L are read
// once.
//
// A work unit is (128-row weight tile, part s of S), S >= 2. The k-stages of a tile (the FP4
// stages, then the compensation stages of B * W_L) are dealt out in S equal runs, so S x tiles
// CTAs stream weights at once instead of one per tile. Each unit writes its fp32 partial
// (M x 128) to a caller-provided workspace and a second kernel, chained by programmatic
// dependent launch, adds the S partials in the order s = 0 .. S-1 and rounds to bf16, so the
// result does not depend on timing.
//
// Roles (256 threads): warp 0 lane 0 TMA producer; warp 1 lane 0 MMA issuer; warp 2 TMEM
// allocator; warp 3 lane 0 scale copier; warps 4..7 epilogue, warp w reading TMEM lanes
// 32 (w % 4) .. + 31 (weight rows).
#include "osc_device.cuh"
#include "osc_internal.h"

namespace osc {

template <int NT, int KIND>
struct SmallCfg {
  static constexpr bool FP8 = KIND == KIND_MXF8_B32;
  static constexpr int V = KIND == KIND_MXF4_B16 ? 16 : 32;
  static constexpr int ELEMS = FP8 ? 128 : 256;                 // K elements per stage (128 bytes a row)
  static constexpr int APS = ELEMS / (4 * V);                   // scale atoms per stage and operand
  static constexpr int SC = SMALL_CHUNK_ATOMS / APS;            // FP4/FP8 stages per scale chunk
  static constexpr int A_BYTES = 128 * 128;                     // weight tile: 128 rows x 128 bytes
  static constexpr int B_BYTES = NT * 128;                      // token tile: NT rows x 128 bytes
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;         // a multiple of 1 KB
  static constexpr int CHUNK_OP_BYTES = SMALL_CHUNK_ATOMS * 512;
  static constexpr int CHUNK_BYTES = 2 * CHUNK_OP_BYTES;        // weight atoms, then token atoms
  static constexpr int CHUNKS = 2;                              // scale chunk buffers
  static constexpr int BAR_BYTES = 1024;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int STAGES_FIT = (SMEM_LIMIT - BAR_BYTES - 1024 - CHUNKS * CHUNK_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
  static constexpr int SMEM_TOTAL = STAGES * STAGE_BYTES + CHUNKS * CHUNK_BYTES + BAR_BYTES + 1024;
  static constexpr int ACC_COLS = NT < 32 ? 32 : NT;            // one accumulator (TMEM columns)
  static constexpr int CHUNK_COLS = 2 * SMALL_CHUNK_ATOMS * 4;  // TMEM columns of one chunk's scales
  static constexpr int SF_COL = 2 * ACC_COLS;                   // two accumulators, then the chunks
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t DATA_TX = A_BYTES + B_BYTES;        // every stage (FP4 and compensation)
  static constexpr int IN_FLIGHT = 4;                           // stage loads outstanding at most
  static_assert(SF_COL + CHUNKS * CHUNK_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(STAGES >= 3, "smem budget");
  static_assert(SC >= 1 && SC * APS == SMALL_CHUNK_ATOMS, "chunk of whole stages");
  static_assert(NT == 16, "token tile: one 16-row MMA N");
};

// Stage range [i0, i1) of unit (tile, s) among T = FP4 stages + compensation stages.
__device__ __forceinline__ void unit_range(int s, int S, int T, int& i0, int& i1) {
  i0 = (int)((long long)s * T / S);
  i1 = (int)((long long)(s + 1) * T / S);
}

constexpr int SMALL_THREADS = 256;

// The scales of a unit's block-scaled stages come in chunks of SC stages (SMALL_CHUNK_ATOMS
// atoms per operand, one TMA box each), double-buffered in shared memory and TMEM: one thread
// copies a whole chunk into TMEM back to back and publishes it once, so the MMA issuer waits
// for scales once per chunk instead of once per stage, and the per-stage ring carries only the
// operand tiles.
template <int NT, int KIND>
__global__ void __launch_bounds__(SMALL_THREADS, 1)
gemm_small_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmSW, const __grid_constant__ CUtensorMap tmSX,
                  const __grid_constant__ CUtensorMap tmWL, const __grid_constant__ CUtensorMap tmB,
                  const SmallParams p) {
  using C = SmallCfg<NT, KIND>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  const uint32_t schunk0 = sbase + C::STAGES * C::STAGE_BYTES;            // chunk buffers
  uint8_t* bar_area = smem + C::STAGES * C::STAGE_BYTES + C::CHUNKS * C::CHUNK_BYTES;
  const uint32_t bar0 = smem_u32(bar_area);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto cfull_bar = [&](int c) { return bar0 + 8u * (2 * C::STAGES + c); };       // chunk landed
  auto cready_bar = [&](int c) { return bar0 + 8u * (2 * C::STAGES + 2 + c); };  // chunk in TMEM
  auto cempty_bar = [&](int c) { return bar0 + 8u * (2 * C::STAGES + 4 + c); };  // chunk's MMAs done
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 6 + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 8 + a); };
  auto tear_bar = [&](int i) { return bar0 + 8u * (2 * C::STAGES + 10 + i); };  // 2 of them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_area + 8 * (2 * C::STAGES + 12));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 8 * (2 * C::STAGES + 12) + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_k = p.K / C::ELEMS;
  const int n_c = (p.K_L + 63) / 64;
  const int T = n_k + n_c;
  const int units = p.n_tiles * p.S;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int c = 0; c < C::CHUNKS; ++c) { mbar_init(cfull_bar(c), 1); mbar_init(cready_bar(c), 1); mbar_init(cempty_bar(c), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(accf_bar(a), 1); mbar_init(acce_bar(a), 4); }
    for (int i = 0; i < 2; ++i) mbar_init(tear_bar(i), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmW); tma_prefetch_desc(&tmX); tma_prefetch_desc(&tmSW); tma_prefetch_desc(&tmSX);
    if (p.K_L > 0) { tma_prefetch_desc(&tmWL); tma_prefetch_desc(&tmB); }
  }
  if (warp == 2) { tc_alloc<1>(smem_u32(tmem_slot), C::TMEM_COLS); tc_relinquish<1>(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) grid_dep_launch();   // the split's reduction may be scheduled now
  grid_dep_wait();                           // Q_X, S_X and B of the previous kernel are visible

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------------ TMA producer
    int stage = 0; uint32_t phase = 0;
    int cb = 0; uint32_t cphase = 0;
    long long fills = 0, cfills = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int tile = u / p.S, s = u % p.S, n0 = tile * 128;
      int i0, i1;
      unit_range(s, p.S, T, i0, i1);
      for (int i = i0; i < i1; ++i) {
        if (i < n_k && (i - i0) % C::SC == 0) {
          // the scale chunk of stages i .. i + SC - 1 (atoms past the unit's range are unused)
          if (!(ok = mbar_wait(cempty_bar(cb), cphase ^ 1, abort_flag, p.status))) break;
          const uint32_t dst = schunk0 + cb * C::CHUNK_BYTES;
          mbar_arrive_expect_tx(cfull_bar(cb), C::CHUNK_BYTES);
          tma_load_3d(dst, &tmSW, 0, i * C::APS, n0 / 128, cfull_bar(cb));
          tma_load_3d(dst + C::CHUNK_OP_BYTES, &tmSX, 0, i * C::APS, 0, cfull_bar(cb));
          ++cfills;
          if (++cb == C::CHUNKS) { cb = 0; cphase ^= 1; }
        }
        if (!(ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, p.status))) break;
        if (fills >= C::IN_FLIGHT) {
          // at most IN_FLIGHT stages requested and not yet landed: every CTA streams weights at
          // once, and a shorter queue lands each CTA's first stages sooner (QKV weights, M = 1:
          // 7.96 vs 8.2 us)
          const long long f = fills - C::IN_FLIGHT;
          if (!(ok = mbar_wait(full_bar((int)(f % C::STAGES)), (uint32_t)((f / C::STAGES) & 1), abort_flag, p.status))) break;
        }
        const uint32_t st = sbase + stage * C::STAGE_BYTES;
        const uint32_t fb = full_bar(stage);
        mbar_arrive_expect_tx(fb, C::DATA_TX);
        if (i < n_k) {
          tma_load_2d(st, &tmW, i * 128, n0, fb);
          tma_load_2d(st + C::A_BYTES, &tmX, i * 128, 0, fb);
        } else {
          const int c = i - n_k;
          tma_load_2d(st, &tmWL, c * 64, n0, fb);
          tma_load_2d(st + C::A_BYTES, &tmB, c * 64, 0, fb);
        }
        ++fills;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (*abort_flag) {
      // let the copies armed on this CTA's barriers land before the CTA exits
      volatile int never = 0;
      const long long last = fills < C::STAGES ? fills : C::STAGES;
      for (long long f = fills - last; f < fills; ++f)
        mbar_wait(full_bar((int)(f % C::STAGES)), (uint32_t)((f / C::STAGES) & 1), &never, nullptr, 100000000ull);
      const long long clast = cfills < C::CHUNKS ? cfills : C::CHUNKS;
      for (long long f = cfills - clast; f < cfills; ++f)
        mbar_wait(cfull_bar((int)(f % C::CHUNKS)), (uint32_t)((f / C::CHUNKS) & 1), &never, nullptr, 100000000ull);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    int stage = 0; uint32_t phase = 0;
    int cb = 0; uint32_t cphase = 0;
    int acc = 0; uint32_t aphase = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int s = u % p.S;
      int i0, i1;
      unit_range(s, p.S, T, i0, i1);
      const int fp_end = min(i1, n_k);                        // the unit's block-scaled stages end here
      if (!(ok = mbar_wait(acce_bar(acc), aphase ^ 1, abort_flag, p.status))) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * C::ACC_COLS;
      bool first = true;
      for (int i = i0; i < i1; ++i) {
        const int in_chunk = (i - i0) % C::SC;
        if (i < n_k && in_chunk == 0) {
          if (!(ok = mbar_wait(cready_bar(cb), cphase, abort_flag, p.status))) break;   // scales in TMEM
        }
        if (!(ok = mbar_wait(full_bar(stage), phase, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t st = sbase + stage * C::STAGE_BYTES;
        if (i < n_k) {
          const uint32_t sfw = tmem + C::SF_COL + cb * C::CHUNK_COLS + in_chunk * C::APS * 4;
          const uint32_t sfx = sfw + SMALL_CHUNK_ATOMS * 4;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t ad = desc_kmajor_sw128(st + 32 * j);
            const uint64_t bd = desc_kmajor_sw128(st + C::A_BYTES + 32 * j);
            const uint32_t accum = first ? 0u : 1u;
            first = false;
            if constexpr (KIND == KIND_MXF4_B32) {
              const uint32_t sf = 2 * (j & 1), atom = j >> 1;
              tc_mma_mxf4_b32_g<1>(d, ad, bd, idesc_bs_m(FMT_MXF4_E2M1, 128, NT, sf, sf),
                                   sfw + 4 * atom, sfx + 4 * atom, accum);
            } else if constexpr (KIND == KIND_MXF4_B16) {
              tc_mma_mxf4_b16_g<1>(d, ad, bd, idesc_bs_m(FMT_MXF4_E2M1, 128, NT, 0, 0), sfw + 4 * j, sfx + 4 * j, accum);
            } else {
              tc_mma_mxf8_g<1>(d, ad, bd, idesc_bs_m(FMT_F8_E4M3, 128, NT, j, j), sfw, sfx, accum);
            }
          }
          tc_commit_to<1>(empty_bar(stage));
          if (in_chunk == C::SC - 1 || i == fp_end - 1) {     // the chunk's MMAs are all issued
            tc_commit_to<1>(cempty_bar(cb));
            if (++cb == C::CHUNKS) { cb = 0; cphase ^= 1; }
          }
        } else {
          const int c = i - n_k;
          const int nm = min(4, (p.K_L - 64 * c) / 16);
          for (int j = 0; j < nm; ++j) {
            tc_mma_bf16_g<1>(d, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + C::A_BYTES + 32 * j),
                             idesc_bf16_m(128, NT), first ? 0u : 1u);
            first = false;
          }
          tc_commit_to<1>(empty_bar(stage));
        }
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      tc_commit_to<1>(accf_bar(acc));
      acc ^= 1;
      if (acc == 0) aphase ^= 1;
    }
    if (*abort_flag) {
      tc_commit_to<1>(tear_bar(0));
      volatile int never = 0;
      mbar_wait(tear_bar(0), 0, &never, nullptr, 100000000ull);
    }
  } else if (warp == 3 && lane == 0) {
    // ------------------------------------------------------------------ scale copier
    // a chunk's TMEM set is free again once its smem buffer is refilled: the producer reloads
    // a buffer only after the MMAs that read the previous chunk there have completed
    int cb = 0; uint32_t cphase = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int s = u % p.S;
      int i0, i1;
      unit_range(s, p.S, T, i0, i1);
      const int n_fp = max(0, min(i1, n_k) - i0);
      for (int c = 0; c < (n_fp + C::SC - 1) / C::SC; ++c) {
        if (!(ok = mbar_wait(cfull_bar(cb), cphase, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t src = schunk0 + cb * C::CHUNK_BYTES;
        const uint32_t dst = tmem + C::SF_COL + cb * C::CHUNK_COLS;
        const int atoms = min(C::SC, n_fp - c * C::SC) * C::APS;   // the atoms the chunk's MMAs read
        for (int a = 0; a < atoms; ++a) {
          tc_cp_atom<1>(dst + 4 * a, desc_scale_atom(src + 512 * a));
          tc_cp_atom<1>(dst + SMALL_CHUNK_ATOMS * 4 + 4 * a, desc_scale_atom(src + C::CHUNK_OP_BYTES + 512 * a));
        }
        tc_commit_local<1>(cready_bar(cb));
        if (++cb == C::CHUNKS) { cb = 0; cphase ^= 1; }
      }
    }
    if (*abort_flag) {
      tc_commit_local<1>(tear_bar(1));
      volatile int never = 0;
      mbar_wait(tear_bar(1), 0, &never, nullptr, 100000000ull);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                                  // TMEM lanes 32q .. 32q + 31
    int acc = 0; uint32_t aphase = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const int tile = u / p.S, s = u % p.S;
      if (!mbar_wait(accf_bar(acc), aphase, abort_flag, p.status)) break;
      tc_fence_after();
      const int n = tile * 128 + 32 * q + lane;               // this thread's weight row = output column
      const bool col_ok = n < p.N;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + acc * C::ACC_COLS;
      uint32_t r[NT];
      tmem_ld16(tbase, r);                                     // the NT = 16 token columns
      tmem_ld_wait();
      if (col_ok) {
#pragma unroll
        for (int m = 0; m < NT; ++m)
          if (m < p.M) p.partial[((size_t)s * p.M + m) * p.N + n] = __uint_as_float(r[m]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(acc));
      acc ^= 1;
      if (acc == 0) aphase ^= 1;
    }
  }

  tc_fence_before();
  __syncwarp();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tc_dealloc<1>(tmem, C::TMEM_COLS);
  }
}

// Y[m][n] = bf16(sum over s = 0 .. S-1, in that order, of partial[s][m][n]); four columns a
// thread (N is a multiple of 16).
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ partial, int S, int M, int N,
                                                            uint16_t* __restrict__ Y, float* __restrict__ Yf32) {
  grid_dep_wait();                                           // the partials are complete
  if (threadIdx.x == 0) grid_dep_launch();
  const size_t quads = (size_t)M * N / 4;
  for (size_t qd = (size_t)blockIdx.x * blockDim.x + threadIdx.x; qd < quads; qd += (size_t)gridDim.x * blockDim.x) {
    float4 acc = __ldg(reinterpret_cast<const float4*>(partial) + qd);
    for (int s = 1; s < S; ++s) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(partial + (size_t)s * M * N) + qd);
      acc.x = __fadd_rn(acc.x, v.x); acc.y = __fadd_rn(acc.y, v.y);
      acc.z = __fadd_rn(acc.z, v.z); acc.w = __fadd_rn(acc.w, v.w);
    }
    const uint32_t lo = pack_bf16x2(acc.x, acc.y), hi = pack_bf16x2(acc.z, acc.w);
    reinterpret_cast<uint2*>(Y)[qd] = make_uint2(lo, hi);
    if (Yf32 != nullptr) reinterpret_cast<float4*>(Yf32)[qd] = acc;
  }
}

template <int NT, int KIND>
static cudaError_t launch_small_one(const SmallMaps& m, const SmallParams& p, int grid, cudaStream_t s) {
  using C = SmallCfg<NT, KIND>;
  static PerDeviceOnce smem_attr;
  const cudaError_t ae = smem_attr.run([] {
    return cudaFuncSetAttribute(gemm_small_kernel<NT, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_TOTAL);
  });
  if (ae != cudaSuccess) return ae;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(SMALL_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_TOTAL;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_small_kernel<NT, KIND>, m.w, m.x, m.sw, m.sx, m.wl, m.b, p);
}

cudaError_t launch_gemm_small(int kind, const SmallMaps& maps, const SmallParams& p, int grid, cudaStream_t s) {
  if (p.M < 1 || p.M > SPLIT_MAX_M || p.S < 2 || p.partial == nullptr) return cudaErrorInvalidValue;
  cudaError_t e;
  if (kind == KIND_MXF4_B32) e = launch_small_one<SPLIT_MAX_M, KIND_MXF4_B32>(maps, p, grid, s);
  else if (kind == KIND_MXF4_B16) e = launch_small_one<SPLIT_MAX_M, KIND_MXF4_B16>(maps, p, grid, s);
  else if (kind == KIND_MXF8_B32) e = launch_small_one<SPLIT_MAX_M, KIND_MXF8_B32>(maps, p, grid, s);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  // the reduction: a grid of at most 2 x SMs CTAs, chained to the product by programmatic
  // dependent launch so that it is scheduled while the product runs
  const size_t quads = (size_t)p.M * p.N / 4;
  const int rgrid = (int)std::max<size_t>(1, std::min<size_t>((quads + 255) / 256, (size_t)2 * p.num_sms));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rgrid, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, (const float*)p.partial, p.S, p.M, p.N, p.Y, p.Yf32);
}

}  // namespace osc
