// OSC dual-path linear on the sm_100a tensor cores:
//
//   Y = (Q_X (x) Q_W) * S  +  B * W_L
//
// the equation of the OSC page ("W4A4量化技术：OSC框架如何实现高效LLM部署",
// coreui.cn/article/2607942.html), §3.2: a 4-bit base path (block-scaled MXFP4, E8M0 scales)
// plus a 16-bit compensation path for the table's outlier channels. Both run in one kernel:
// the compensation tiles (B: 128 x 64 bf16, W_L: rows x 64 bf16) flow through the same TMA
// ring as the FP4 tiles (both are 128-byte rows) and their kind::f16 MMAs accumulate into the
// same TMEM accumulator right after the FP4 k-loop, so B * W_L costs no extra pass over Y.
// The same kernel serves the MXFP8 fallback of §4 (E4M3 x E4M3, per-32 E8M0) and the
// per-expert grouped form for MoE layers.
//
// Structure: persistent CTAs (one per SM), 12 warps.
//   warp 0 (one lane)   TMA producer: operand tiles (128B swizzle) and scale atoms
//   warp 1 (one lane)   MMA issuer: tcgen05.mma, tcgen05.commit
//   warp 2              TMEM allocator, then (one lane) scale copier of odd stages
//   warp 3 (one lane)   scale copier of even stages: tcgen05.cp of a stage's scale atoms into
//                       that stage's own TMEM scale set; copies issued by threads other than
//                       the MMA issuer overlap the MMAs instead of queueing in front of them
//   warps 4..11         epilogue, two warps per TMEM lane quadrant (warp % 4), each owning half
//                       of the accumulator columns: tcgen05.ld them 64 columns per round trip,
//                       release the accumulator, then bf16 -> smem -> TMA store
// With GemmParams::preload (set only when the kernel before it on the stream is the library's
// own quantize) the producer issues the weight halves of its first tile's first stages before
// griddepcontrol.wait.
// CG = 2 runs the CTA pair of a 2-CTA cluster as one M = 256 tile: each CTA loads its 128
// rows of A and half of the BN rows of B, the leader issues cta_group::2 MMAs over both
// CTAs' shared memory, and each CTA's TMEM holds its 128 rows of the accumulator. Per SM this
// halves the B traffic of a 128 x BN tile for the same tensor work.
// Scales live in TMEM as the block-scaled MMA expects: a 512-byte atom (128 rows x 4 slots)
// is copied with tcgen05.cp 32x128b.warpx4 into 4 columns; row r's slot s is byte s%4 of
// column (r / 32) of its atom; the MMA's scale-factor id picks the byte.
#include "osc_device.cuh"
#include "osc_internal.h"

namespace osc {

template <int BN, int KIND, int CG>
struct GemmCfg {
  static constexpr bool FP8 = KIND == KIND_MXF8_B32;
  static constexpr int V = KIND == KIND_MXF4_B16 ? 16 : 32;        // scale slot width
  static constexpr int ELEMS = FP8 ? 128 : 256;                      // K elements per stage (128 bytes)
  static constexpr int APS = ELEMS / (4 * V);                        // scale atoms per stage
  static constexpr int MMA_M = 128 * CG;
  static constexpr int BROWS = BN / CG;                              // B rows this CTA loads
  static constexpr int A_BYTES = 128 * 128;
  static constexpr int B_BYTES = BROWS * 128;
  static constexpr int SFA_BYTES = APS * 512;
  static constexpr int SFB_BYTES = (BN / 128) * APS * 512;           // every CTA holds all BN rows
  static constexpr int STAGE_RAW = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGE_BYTES = (STAGE_RAW + 1023) / 1024 * 1024;
  static constexpr int EPI_WARPS = 8;                                // two per TMEM lane quadrant
  static constexpr int EPI_COLS = BN / 2;                            // accumulator columns per epilogue warp
  static constexpr int STAGING_BYTES = EPI_WARPS * 32 * 32;          // one 32x16 bf16 tile per epilogue warp
  static constexpr int BAR_BYTES = 1024;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int STAGES_FIT = (SMEM_LIMIT - STAGING_BYTES - BAR_BYTES - 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM_TOTAL = STAGES * STAGE_BYTES + STAGING_BYTES + BAR_BYTES + 1024;
  static constexpr int SFA_COLS = APS * 4;
  static constexpr int SFB_COLS = APS * (BN / 32);
  static constexpr int SF_SET = SFA_COLS + SFB_COLS;                 // TMEM columns of one stage's scales
  static constexpr int ACC_STAGES = (2 * BN + STAGES * SF_SET <= 512) ? 2 : 1;
  static constexpr int SFA_COL = ACC_STAGES * BN;                    // scale set s starts at SFA_COL + s * SF_SET
  static constexpr int SFB_COL = SFA_COL + SFA_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t MAIN_TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;   // per CTA and stage
  static constexpr uint32_t COMP_TX = A_BYTES + B_BYTES;
  static_assert(SFA_COL + STAGES * SF_SET <= TMEM_COLS, "TMEM budget");
  static_assert(STAGES >= 2, "smem budget");
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "tile width");
  static_assert(CG == 1 || (CG == 2 && BN == 256), "the CTA pair uses 256-wide tiles");
};

struct TileInfo {
  int m0, n0, e, kl;   // m0: this CTA's first row
};

// Tile order: dense products walk the row blocks fastest (CTAs running together share a
// weight tile; at these sizes every operand fits L2 anyway). Grouped products walk the column
// blocks fastest: CTAs running together then work on one expert's row block (sharing its
// activation tile), and an expert's next row block follows right after, while its weights are
// still in L2; row blocks fastest would spread concurrent CTAs over many experts and evict
// each expert's weights between its row blocks.
template <int CG>
__device__ __forceinline__ TileInfo tile_info(int t, const GemmParams& p, int bn, int rank) {
  TileInfo ti;
  const bool by_row = p.num_groups != 0;
  const int mb = by_row ? t / p.n_tiles : t % p.m_tiles;   // m_tiles counts (128 * CG)-row tiles
  const int nb = by_row ? t % p.n_tiles : t / p.m_tiles;
  ti.m0 = mb * 128 * CG + 128 * rank;
  ti.n0 = nb * bn;
  if (p.num_groups == 0) {
    ti.e = 0;
    ti.kl = p.K_L;
  } else {
    ti.e = __ldg(p.mblock_expert + mb);
    ti.kl = p.group_kl ? __ldg(p.group_kl + ti.e) : p.K_L;
  }
  return ti;
}

constexpr int GEMM_THREADS = 384;

template <int BN, int KIND, int CG>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
            const __grid_constant__ CUtensorMap tmCA, const __grid_constant__ CUtensorMap tmCB,
            const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  using C = GemmCfg<BN, KIND, CG>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_addr + pad;
  const uint32_t s_staging = sbase + C::STAGES * C::STAGE_BYTES;
  uint8_t* bar_area = smem + C::STAGES * C::STAGE_BYTES + C::STAGING_BYTES;
  const uint32_t bar0 = smem_u32(bar_area);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 2 + a); };
  const uint32_t tear_bar = bar0 + 8u * (2 * C::STAGES + 4);
  const uint32_t tear2_bar = bar0 + 8u * (2 * C::STAGES + 5);
  auto sfready_bar = [&](int s) { return bar0 + 8u * (2 * C::STAGES + 6 + s); };
  const uint32_t tear3_bar = bar0 + 8u * (3 * C::STAGES + 6);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_area + 8 * (3 * C::STAGES + 7));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_area + 8 * (3 * C::STAGES + 7) + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = CG == 2 ? (int)cluster_ctarank() : 0;
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(accf_bar(a), 1); mbar_init(acce_bar(a), C::EPI_WARPS * CG); }
    mbar_init(tear_bar, 1);
    mbar_init(tear2_bar, 1);
    mbar_init(tear3_bar, 1);
    for (int s = 0; s < C::STAGES; ++s) mbar_init(sfready_bar(s), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB); tma_prefetch_desc(&tmY);
    tma_prefetch_desc(&tmSFA); tma_prefetch_desc(&tmSFB);
    if (p.K_L > 0) { tma_prefetch_desc(&tmCA); tma_prefetch_desc(&tmCB); }
  }
  if (warp == 2) { tc_alloc<CG>(smem_u32(tmem_slot), C::TMEM_COLS); tc_relinquish<CG>(); }
  tc_fence_before();
  __syncwarp();                          // the cluster barrier below is warp-aligned
  if constexpr (CG == 2) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int num_tiles = p.m_tiles * p.n_tiles;
  const int n_k = p.K / C::ELEMS;
  const int n_rb = (p.N + 127) / 128;
  const int unit = blockIdx.x / CG, nunits = gridDim.x / CG;
  // With p.preload the producer issues the weight parts (B and its scales) of its first tile's
  // first stages before the dependency wait, so they stream in while the previous kernel (the
  // library's own quantize of X, which writes no weights) finishes; the activation parts follow
  // after the wait. A stage's full barrier counts both parts.
  int pre = 0;
  if (warp == 0 && lane == 0 && p.preload && p.num_groups == 0 && unit < num_tiles) {
    const TileInfo ti = tile_info<CG>(unit, p, BN, rank);   // dense: no device memory read
    const int brow = ti.n0 + rank * C::BROWS;
    pre = min(C::STAGES, n_k);
    for (int ks = 0; ks < pre; ++ks) {
      const uint32_t st = sbase + ks * C::STAGE_BYTES;
      if constexpr (CG == 1) {
        const uint32_t fb = full_bar(ks);
        mbar_arrive_expect_tx(fb, C::MAIN_TX);
        tma_load_3d(st + C::A_BYTES, &tmB, ks * 128, brow, 0, fb);
        tma_load_3d(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSFB, 0, ks * C::APS, ti.n0 / 128, fb);
      } else {
        const uint32_t fb = mapa_shared(full_bar(ks), 0);
        if (leader) mbar_arrive_expect_tx(full_bar(ks), 2 * C::MAIN_TX);
        tma_load_3d_pair(st + C::A_BYTES, &tmB, ks * 128, brow, 0, fb);
        tma_load_3d_pair(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSFB, 0, ks * C::APS, ti.n0 / 128, fb);
      }
    }
  }
  grid_dep_wait();                       // the previous kernel's writes (Q_X, S_X, B) are visible
  if (threadIdx.x == 0) grid_dep_launch();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------------ TMA producer
    int stage = 0; uint32_t phase = 0;
    long long fills = 0;
    for (int t = unit; t < num_tiles; t += nunits) {
      const TileInfo ti = tile_info<CG>(t, p, BN, rank);
      const int brow = ti.n0 + rank * C::BROWS;
      bool ok = true;
      for (int ks = 0; ks < n_k && ok; ++ks) {
        if (!(ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, p.status))) break;
        const uint32_t st = sbase + stage * C::STAGE_BYTES;
        const bool w_issued = t == unit && ks < pre;            // weight parts issued before the wait
        if constexpr (CG == 1) {
          const uint32_t fb = full_bar(stage);
          if (!w_issued) mbar_arrive_expect_tx(fb, C::MAIN_TX);
          tma_load_2d(st, &tmA, ks * 128, ti.m0, fb);
          if (!w_issued) tma_load_3d(st + C::A_BYTES, &tmB, ks * 128, brow, ti.e, fb);
          tma_load_3d(st + C::A_BYTES + C::B_BYTES, &tmSFA, 0, ks * C::APS, ti.m0 / 128, fb);
          if (!w_issued)
            tma_load_3d(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSFB, 0, ks * C::APS,
                        ti.e * n_rb + ti.n0 / 128, fb);
        } else {
          const uint32_t fb = mapa_shared(full_bar(stage), 0);     // the leader counts both CTAs' bytes
          if (leader && !w_issued) mbar_arrive_expect_tx(full_bar(stage), 2 * C::MAIN_TX);
          tma_load_2d_pair(st, &tmA, ks * 128, ti.m0, fb);
          if (!w_issued) tma_load_3d_pair(st + C::A_BYTES, &tmB, ks * 128, brow, ti.e, fb);
          tma_load_3d_pair(st + C::A_BYTES + C::B_BYTES, &tmSFA, 0, ks * C::APS, ti.m0 / 128, fb);
          if (!w_issued)
            tma_load_3d_pair(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSFB, 0, ks * C::APS,
                             ti.e * n_rb + ti.n0 / 128, fb);
        }
        ++fills;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      const int n_c = (ti.kl + 63) / 64;
      for (int c = 0; c < n_c && ok; ++c) {
        if (!(ok = mbar_wait(empty_bar(stage), phase ^ 1, abort_flag, p.status))) break;
        const uint32_t st = sbase + stage * C::STAGE_BYTES;
        if constexpr (CG == 1) {
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, C::COMP_TX);
          tma_load_2d(st, &tmCA, c * 64, ti.m0, fb);
          tma_load_3d(st + C::A_BYTES, &tmCB, c * 64, brow, ti.e, fb);
        } else {
          const uint32_t fb = mapa_shared(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * C::COMP_TX);
          tma_load_2d_pair(st, &tmCA, c * 64, ti.m0, fb);
          tma_load_3d_pair(st + C::A_BYTES, &tmCB, c * 64, brow, ti.e, fb);
        }
        ++fills;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    if (*abort_flag && leader) {
      // let the copies armed on this CTA's barriers land before the CTA exits
      const long long last = fills < C::STAGES ? fills : C::STAGES;
      for (long long f = fills - last; f < fills; ++f) {
        volatile int never = 0;
        mbar_wait(full_bar((int)(f % C::STAGES)), (uint32_t)((f / C::STAGES) & 1), &never, nullptr, 100000000ull);
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------------ MMA issuer
    int stage = 0; uint32_t phase = 0;
    int acc = 0; uint32_t aphase = 0;
    bool ok = true;
    for (int t = unit; t < num_tiles && ok; t += nunits) {
      const TileInfo ti = tile_info<CG>(t, p, BN, rank);
      if (!(ok = mbar_wait(acce_bar(acc), aphase ^ 1, abort_flag, p.status))) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * BN;
      for (int ks = 0; ks < n_k; ++ks) {
        // the stage's operands landed and its scales are in TMEM
        if (!(ok = mbar_wait2(full_bar(stage), sfready_bar(stage), phase, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t st = sbase + stage * C::STAGE_BYTES;
        const uint32_t sfo = tmem + stage * C::SF_SET;      // this stage's scale set
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t ad = desc_kmajor_sw128(st + 32 * j);
          const uint64_t bd = desc_kmajor_sw128(st + C::A_BYTES + 32 * j);
          const uint32_t accum = (ks > 0 || j > 0) ? 1u : 0u;
          if constexpr (KIND == KIND_MXF4_B32) {
            const uint32_t sf = 2 * (j & 1), atom = j >> 1;
            tc_mma_mxf4_b32_g<CG>(d, ad, bd, idesc_bs_m(FMT_MXF4_E2M1, C::MMA_M, BN, sf, sf),
                                  sfo + C::SFA_COL + 4 * atom, sfo + C::SFB_COL + atom * (BN / 32), accum);
          } else if constexpr (KIND == KIND_MXF4_B16) {
            tc_mma_mxf4_b16_g<CG>(d, ad, bd, idesc_bs_m(FMT_MXF4_E2M1, C::MMA_M, BN, 0, 0),
                                  sfo + C::SFA_COL + 4 * j, sfo + C::SFB_COL + j * (BN / 32), accum);
          } else {
            tc_mma_mxf8_g<CG>(d, ad, bd, idesc_bs_m(FMT_F8_E4M3, C::MMA_M, BN, j, j),
                              sfo + C::SFA_COL, sfo + C::SFB_COL, accum);
          }
        }
        tc_commit_to<CG>(empty_bar(stage));
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      const int n_c = (ti.kl + 63) / 64;
      for (int c = 0; c < n_c && ok; ++c) {
        // (the compensation stages' scale barrier carries no scales; waiting on it keeps phases aligned)
        if (!(ok = mbar_wait2(full_bar(stage), sfready_bar(stage), phase, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t st = sbase + stage * C::STAGE_BYTES;
        const int nm = min(4, (ti.kl - 64 * c) / 16);
        for (int j = 0; j < nm; ++j)
          tc_mma_bf16_g<CG>(d, desc_kmajor_sw128(st + 32 * j), desc_kmajor_sw128(st + C::A_BYTES + 32 * j),
                            idesc_bf16_m(C::MMA_M, BN), 1u);
        tc_commit_to<CG>(empty_bar(stage));
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      tc_commit_to<CG>(accf_bar(acc));
      if (C::ACC_STAGES == 2) { acc ^= 1; if (acc == 0) aphase ^= 1; } else { aphase ^= 1; }
    }
    if (*abort_flag) {
      tc_commit_to<CG>(tear_bar);
      volatile int never = 0;
      mbar_wait(tear_bar, 0, &never, nullptr, 100000000ull);
    }
  } else if ((warp == 3 || warp == 2) && lane == 0 && leader) {
    // ------------------------------------------------------------------ scale copiers
    // Two copier threads (warps 3 and 2; warp 2 is free once TMEM is allocated) take alternate
    // stages of the sequence the MMA issuer walks: six atom copies take about one stage of MMA
    // time when issued beside running MMAs, so a single copier falls behind. A stage's scale
    // set is free once the stage's data has landed again (the producer refills a stage only
    // after the MMAs that read it - and its scale set - have completed).
    const uint32_t mine = warp == 3 ? 0u : 1u;
    int stage = 0; uint32_t phase = 0;
    uint32_t seq = 0;                                      // position in the stage sequence
    bool ok = true;
    for (int t = unit; t < num_tiles && ok; t += nunits) {
      const TileInfo ti = tile_info<CG>(t, p, BN, rank);
      const int n_c = (ti.kl + 63) / 64;
      for (int i = 0; i < n_k + n_c; ++i, ++seq) {
        if ((seq & 1u) == mine) {
          if (!(ok = mbar_wait(full_bar(stage), phase, abort_flag, p.status))) break;
          if (i < n_k) {
            tc_fence_after();
            const uint32_t s_sfa = sbase + stage * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
            const uint32_t s_sfb = s_sfa + C::SFA_BYTES;
            const uint32_t sfo = tmem + stage * C::SF_SET;
#pragma unroll
            for (int a = 0; a < C::APS; ++a) {
              tc_cp_atom<CG>(sfo + C::SFA_COL + 4 * a, desc_scale_atom(s_sfa + 512 * a));
#pragma unroll
              for (int r = 0; r < BN / 128; ++r)
                tc_cp_atom<CG>(sfo + C::SFB_COL + a * (BN / 32) + 4 * r, desc_scale_atom(s_sfb + (r * C::APS + a) * 512));
            }
            tc_commit_local<CG>(sfready_bar(stage));
          } else {
            mbar_arrive(sfready_bar(stage));               // compensation stages carry no scales
          }
        }
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (*abort_flag) {
      const uint32_t tb = warp == 3 ? tear2_bar : tear3_bar;
      tc_commit_local<CG>(tb);
      volatile int never = 0;
      mbar_wait(tb, 0, &never, nullptr, 100000000ull);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                            // TMEM lane quadrant of this warp
    const int half = (warp - 4) >> 2;                  // which half of the accumulator columns
    const int ew = warp - 4;
    const uint32_t stg = s_staging + ew * (32 * 32);
    uint8_t* stg_ptr = smem + C::STAGES * C::STAGE_BYTES + ew * (32 * 32);
    constexpr int NCH = C::EPI_COLS / 32;              // 32-column chunks per warp (4 or 2)
    int acc = 0; uint32_t aphase = 0;
    for (int t = unit; t < num_tiles; t += nunits) {
      const TileInfo ti = tile_info<CG>(t, p, BN, rank);
      if (!mbar_wait(accf_bar(acc), aphase, abort_flag, p.status)) break;
      tc_fence_after();
      const int row = ti.m0 + 32 * q + lane;
      const int c0 = half * C::EPI_COLS;               // first accumulator column of this warp
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + acc * BN + c0;
      uint32_t packed[C::EPI_COLS / 2];
#pragma unroll
      for (int ch = 0; ch < NCH; ch += 2) {            // two chunks per TMEM round trip
        uint32_t r[2][32];
        tmem_ld32(tbase + ch * 32, r[0]);
        tmem_ld32(tbase + ch * 32 + 32, r[1]);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (p.Yf32 != nullptr && row < p.M) {
            const int col0 = ti.n0 + c0 + (ch + u) * 32;
            float* dst = p.Yf32 + (size_t)row * p.N + col0;
            if (col0 + 32 <= p.N) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                reinterpret_cast<float4*>(dst)[i] = make_float4(__uint_as_float(r[u][4 * i]), __uint_as_float(r[u][4 * i + 1]),
                                                                __uint_as_float(r[u][4 * i + 2]), __uint_as_float(r[u][4 * i + 3]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)         // fully unrolled: r stays in registers
                if (col0 + i < p.N) dst[i] = __uint_as_float(r[u][i]);
            }
          }
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[(ch + u) * 16 + i] = pack_bf16x2(__uint_as_float(r[u][2 * i]), __uint_as_float(r[u][2 * i + 1]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (CG == 1) mbar_arrive(acce_bar(acc));
        else mbar_arrive_cluster(mapa_shared(acce_bar(acc), 0));
      }
      if (C::ACC_STAGES == 2) { acc ^= 1; if (acc == 0) aphase ^= 1; } else { aphase ^= 1; }

      const bool rows_live = ti.m0 + 32 * q < p.M;
#pragma unroll
      for (int cc = 0; cc < 2 * NCH; ++cc) {           // 16-column pieces
        const int col = ti.n0 + c0 + cc * 16;
        if (!rows_live || col >= p.N) continue;        // warp-uniform (N is a multiple of 16)
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        // 32 rows x 32 bytes in the 32-byte swizzle the store map uses: 16-byte chunk c of
        // row r sits at chunk c ^ ((r / 4) % 2)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint4 v = make_uint4(packed[cc * 8 + 4 * i], packed[cc * 8 + 4 * i + 1],
                                     packed[cc * 8 + 4 * i + 2], packed[cc * 8 + 4 * i + 3]);
          *reinterpret_cast<uint4*>(stg_ptr + lane * 32 + ((i ^ ((lane >> 2) & 1)) * 16)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) { tma_store_2d(&tmY, stg, col, ti.m0 + 32 * q); bulk_commit(); }
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncwarp();                          // role lanes rejoin their warps before the aligned barrier
  if constexpr (CG == 2) cluster_sync(); else __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tc_dealloc<CG>(tmem, C::TMEM_COLS);
  }
}

template <int BN, int KIND, int CG>
static cudaError_t launch_one(const GemmMaps& m, const GemmParams& p, int grid, cudaStream_t s) {
  using C = GemmCfg<BN, KIND, CG>;
  static PerDeviceOnce smem_attr;
  const cudaError_t ae = smem_attr.run([] {
    return cudaFuncSetAttribute(gemm_kernel<BN, KIND, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_TOTAL);
  });
  if (ae != cudaSuccess) return ae;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_TOTAL;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_kernel<BN, KIND, CG>, m.a, m.b, m.sfa, m.sfb, m.ca, m.cb, m.y, p);
}

cudaError_t launch_gemm(int kind, int bn, int cg, const GemmMaps& maps, const GemmParams& p, int grid, cudaStream_t s) {
  if (cg == 2) {
    if (bn != 256) return cudaErrorInvalidValue;
    if (kind == KIND_MXF4_B32) return launch_one<256, KIND_MXF4_B32, 2>(maps, p, grid, s);
    if (kind == KIND_MXF4_B16) return launch_one<256, KIND_MXF4_B16, 2>(maps, p, grid, s);
    if (kind == KIND_MXF8_B32) return launch_one<256, KIND_MXF8_B32, 2>(maps, p, grid, s);
    return cudaErrorInvalidValue;
  }
  if (bn == 256) {
    if (kind == KIND_MXF4_B32) return launch_one<256, KIND_MXF4_B32, 1>(maps, p, grid, s);
    if (kind == KIND_MXF4_B16) return launch_one<256, KIND_MXF4_B16, 1>(maps, p, grid, s);
    if (kind == KIND_MXF8_B32) return launch_one<256, KIND_MXF8_B32, 1>(maps, p, grid, s);
  } else if (bn == 128) {
    if (kind == KIND_MXF4_B32) return launch_one<128, KIND_MXF4_B32, 1>(maps, p, grid, s);
    if (kind == KIND_MXF4_B16) return launch_one<128, KIND_MXF4_B16, 1>(maps, p, grid, s);
    if (kind == KIND_MXF8_B32) return launch_one<128, KIND_MXF8_B32, 1>(maps, p, grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace osc
