// Internal declarations shared by the .cu files of libosc.so (not part of the C ABI).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <mutex>

namespace osc {

// One-time, per-device set-up (a kernel attribute) that any number of host threads may reach
// at once: `f` runs once for each device, with that device current, and every caller on that
// device gets the first run's result.
struct PerDeviceOnce {
  static constexpr int kMaxDevices = 64;
  std::once_flag flag[kMaxDevices];
  cudaError_t result[kMaxDevices] = {};
  template <class F>
  cudaError_t run(F f) {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(flag[dev], [&] { result[dev] = f(); });
    return result[dev];
  }
};

// Protected channels per group: a table holds K/G x R entries (R <= MAX_R), slot r of group k
// at L[k * R + r], -1 = none.
constexpr int MAX_R = 3;
// Largest table (K/G x R entries) the dense quantize stages in shared memory.
constexpr int MAX_TAB = 4096;

struct QuantParams {
  const uint16_t* X;   // M x K bf16
  int M, K, G, Kg;
  const int8_t* L;     // Kg x R entries (device) or nullptr for no table
  int R;
  int K_L;
  uint8_t* Q;          // packed codes
  uint8_t* S;          // scales in the MMA layout
  uint16_t* B;         // M x K_L bf16 (table only)
  int* status;
};

// Items (32-channel blocks) per warp step of the quantize kernels = height of the TMA box
// the host encodes for X.
constexpr int QUANT_STEP_ITEMS = 64;
// tmX: X as (32-channel blocks) x 64 bytes, box {32, QUANT_STEP_ITEMS}, 64-byte swizzle
// (see make_block_map)
cudaError_t launch_quantize(const CUtensorMap& tmX, const QuantParams& p, bool fp8, int num_sms, cudaStream_t s);

// Producer-fused quantize: RMSNorm of each row, then the OSC quantize of the normalized row.
struct NormQuantParams {
  const uint16_t* X;       // M x K bf16
  const uint16_t* gamma;   // K bf16
  float eps;
  int M, K, G, Kg;
  const int8_t* L;         // Kg x R entries (device) or nullptr
  int R;
  int K_L;
  uint8_t* Q;
  uint8_t* S;
  uint16_t* B;
  int* status;
};
// largest K of the fused form: two row buffers per warp (2 K bytes each) and gamma in shared memory
constexpr int NQ_MAX_K = 6144;
// tmX: X as (32-channel blocks) x 64 bytes, box {32, K/32} (one row per box), 64-byte swizzle
cudaError_t launch_rmsnorm_quantize(const CUtensorMap& tmX, const NormQuantParams& p, int num_sms, cudaStream_t s);

struct GroupedQuantParams {
  const uint16_t* X;          // off[E] x K bf16, expert-sorted
  const int* off;             // E+1 (device)
  const int* poff;            // E+1 (device)
  const int* mblock_expert;   // Mp/128 (device)
  int E, Mp, K, G, Kg;
  const int8_t* L;            // E x Kg x R (device)
  int R;
  int K_L;
  uint8_t* Q;
  uint8_t* S;
  uint16_t* B;
  int* status;
};
cudaError_t launch_quantize_grouped(const GroupedQuantParams& p, int num_sms, cudaStream_t s);
// TMA form over the T = off[E] routed rows (tmX: the dense kernel's block view of those rows)
cudaError_t launch_quantize_grouped_tma(const CUtensorMap& tmX, const GroupedQuantParams& p, int T, int num_sms,
                                        cudaStream_t s);
size_t grouped_tma_smem(int E, int Kg, int R);
constexpr int GROUPED_TMA_SMEM_MAX = 200 * 1024;
// shared memory the grouped quantize needs to stage every expert's table, and its limit
size_t grouped_quant_smem(int E, int Kg, int R);
constexpr int GROUPED_QUANT_SMEM_MAX = 200 * 1024;
cudaError_t launch_gather_wl(const uint16_t* W, int N, int K, int G, const int8_t* L, int R, int K_L, uint16_t* WL,
                             int* status, int num_sms, cudaStream_t s);

// GEMM operand kinds
enum GemmKind : int { KIND_MXF4_B32 = 0, KIND_MXF4_B16 = 1, KIND_MXF8_B32 = 2 };

struct GemmParams {
  int M, N, K, K_L;
  const uint8_t* SFA;    // activation scales (MMA layout)
  const uint8_t* SFB;    // weight scales (MMA layout)
  int nslot4;            // 512-byte scale atoms per 128-row block = K / V / 4
  int m_tiles, n_tiles;
  float* Yf32;           // optional fp32 copy of the output (tests)
  int* status;
  // grouped (MoE) mode when num_groups > 0: each 128-row block of the (padded) row space
  // belongs to one expert, whose weights are slice e of the 3-D weight maps
  int num_groups;
  const int* mblock_expert;      // m_tiles entries (device)
  const int* group_kl;           // per-expert compensation width (device) or nullptr = K_L
  // 1 (dense calls only): the kernel issued just before on the stream writes no weight operand,
  // so the weight parts of the first tile's stages may be loaded before the dependency wait
  int preload;
};

struct GemmMaps {
  CUtensorMap a, b, sfa, sfb, ca, cb, y;
};

// cg = 1: one CTA per 128-row tile; cg = 2: a 2-CTA cluster per 256-row tile (bn = 256).
// grid is a multiple of cg; m_tiles in p counts (128 * cg)-row tiles.
cudaError_t launch_gemm(int kind, int bn, int cg, const GemmMaps& maps, const GemmParams& p, int grid, cudaStream_t s);

// Few token rows (M <= 128): the transposed product with the weight tile as the 128-row MMA
// operand, split over K into S parts (S > 1: fp32 partials in `partial`, S x M x N, added by a
// chained reduction kernel).
struct SmallParams {
  int M, N, K, K_L;
  int S, n_tiles, num_sms;
  uint16_t* Y;
  float* Yf32;
  float* partial;
  int* status;
};
struct SmallMaps {
  CUtensorMap w, x, sw, sx, wl, b;
};
// The split few-row product serves osc_linear_splitk up to this many token rows (one 16-wide
// token tile). Measured on the B200 at the QKV weights (K = 4096, N = 6144, cold): 8.8 / 9.4 us
// at M = 1 / 16 against 10.1 us for the general kernel, which is as fast or faster from M = 32.
constexpr int SPLIT_MAX_M = 16;
// Scale atoms (512 bytes: 128 rows x 4 slots) one scale chunk of the few-row product holds
// per operand: the host encodes the scale maps with boxes of this many atoms.
constexpr int SMALL_CHUNK_ATOMS = 16;
cudaError_t launch_gemm_small(int kind, const SmallMaps& maps, const SmallParams& p, int grid, cudaStream_t s);

struct TableParams {
  const uint16_t* X;   // S x K bf16
  int S, K, G;
  float alpha;
  int min_hits;
  int R;               // rounds: protected channels per group
  int8_t* L;           // K/G x R
};
cudaError_t launch_build_table(const TableParams& p, int num_sms, cudaStream_t s);

struct DensityParams {
  const uint16_t* X;   // S x K bf16
  int S, K, G;
  float alpha;
  const int8_t* L;     // K/G entries
  int* n_hit;          // K/G
  int* n_total;        // K/G
  int* status;
};
cudaError_t launch_density(const DensityParams& p, cudaStream_t s);

// one bounded wait on a barrier nothing signals: records a timeout in `status`
cudaError_t launch_selftest_wait(int* status, unsigned long long limit_ns, cudaStream_t s);

}  // namespace osc
