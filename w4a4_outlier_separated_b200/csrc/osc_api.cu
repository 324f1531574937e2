// The C ABI of libosc.so (declared in include/osc.h): argument checks, per-device state,
// TMA descriptor encoding and kernel launches. No entry point allocates or frees memory.
#include "osc.h"
#include "osc_device.cuh"
#include "osc_internal.h"

#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

namespace {

thread_local int t_last_cuda = 0;
std::atomic<int> g_tile_n{0};
std::atomic<int> g_pair{-1};   // -1 automatic, 1 single CTAs, 2 CTA pairs

__device__ int g_status_word;   // per-device error word written by the kernels
__device__ int g_status_taken;  // where osc_status's exchange leaves the word's old value

// Reads and clears the status word in one atomic step, so an error recorded by a kernel on
// another stream is either returned now or left for the next read, never lost in between.
__global__ void status_take_kernel() { g_status_taken = atomicExch(&g_status_word, 0); }

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  bool sm100 = false;
  int sms = 0;
  int* status = nullptr;
  int* taken = nullptr;   // device address of g_status_taken
  std::mutex status_mu;   // one osc_status at a time per device in this process
};

int fail_cuda(cudaError_t e) {
  t_last_cuda = (int)e;
  return OSC_ERR_CUDA;
}

// Per-device facts, looked up once per device with that device current.
int device_state(DeviceState** out) {
  static std::mutex mu;
  static DeviceState states[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return OSC_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  DeviceState& s = states[dev];
  if (!s.ready) {
    int major = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return fail_cuda(e);
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return fail_cuda(e);
    void* addr = nullptr;
    void* taken = nullptr;
    if ((e = cudaGetSymbolAddress(&addr, g_status_word)) != cudaSuccess) return fail_cuda(e);
    if ((e = cudaGetSymbolAddress(&taken, g_status_taken)) != cudaSuccess) return fail_cuda(e);
    s.sm100 = (major == 10);
    s.sms = sms;
    s.status = static_cast<int*>(addr);
    s.taken = static_cast<int*>(taken);
    s.ready = true;
  }
  if (!s.sm100) return OSC_ERR_DEVICE;
  *out = &s;
  return OSC_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tiled TMA descriptor over a row-major tensor; dims[0] is the contiguous dimension.
int make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
             const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return fail_cuda(cudaErrorNotSupported);
  uint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides), reinterpret_cast<const cuuint32_t*>(box),
                  reinterpret_cast<const cuuint32_t*>(es), CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail_cuda(cudaErrorInvalidValue);
  return OSC_OK;
}

inline bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// X (rows x K bf16) seen by the quantize kernels as 32-channel blocks: 2-D {32, rows*K/32},
// 64-byte rows, box {32, 64}, 64-byte swizzle.
int make_block_map(CUtensorMap* m, const uint16_t* X, int rows, int K) {
  uint64_t d[2] = {32, (uint64_t)rows * (uint64_t)(K / 32)}, st[1] = {64};
  uint32_t box[2] = {32, (uint32_t)osc::QUANT_STEP_ITEMS};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, d, st, box, CU_TENSOR_MAP_SWIZZLE_64B);
}
// The same view with one whole row per box (box {32, K/32}): the fused RMSNorm form.
int make_row_map(CUtensorMap* m, const uint16_t* X, int rows, int K) {
  uint64_t d[2] = {32, (uint64_t)rows * (uint64_t)(K / 32)}, st[1] = {64};
  uint32_t box[2] = {32, (uint32_t)(K / 32)};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, d, st, box, CU_TENSOR_MAP_SWIZZLE_64B);
}
inline bool valid_g(int G) { return G == 16 || G == 32 || G == 64; }

int launch_result(cudaError_t e) { return e == cudaSuccess ? OSC_OK : fail_cuda(e); }

}  // namespace

namespace {

// The split plan of the few-row product: S parts of K per 128-row weight tile, so that
// tiles x S CTAs (at most one per SM) stream the weights. S = 1 (no split: the general kernel
// runs instead) above SPLIT_MAX_M token rows or when the tiles alone fill the SMs.
struct SmallPlan {
  int S, n_tiles;
  size_t partial_bytes;
};
SmallPlan small_plan(int kind, int M, int N, int K, int K_L, int sms) {
  SmallPlan pl;
  pl.n_tiles = (N + 127) / 128;
  const int T = K / (kind == osc::KIND_MXF8_B32 ? 128 : 256) + (K_L + 63) / 64;
  int S = M <= osc::SPLIT_MAX_M ? sms / std::max(1, pl.n_tiles) : 1;
  S = std::max(1, std::min(S, std::min(8, T / 2)));
  pl.S = S;
  pl.partial_bytes = S > 1 ? (size_t)S * (size_t)M * (size_t)N * sizeof(float) : 0;
  return pl;
}

// Split few-row product (M <= SPLIT_MAX_M, dense calls with a workspace that holds the plan's
// partials): see osc_linear_small.cu.
int run_gemm_small(int kind, const uint8_t* QX, const uint8_t* SX, const uint16_t* B, const uint8_t* QW,
                   const uint8_t* SW, const uint16_t* WL, int M, int N, int K, int K_L, uint16_t* Y, float* Yf32,
                   float* workspace, const SmallPlan& pl, const DeviceState* ds, cudaStream_t stream) {
  const bool fp8 = kind == osc::KIND_MXF8_B32;
  const int V = kind == osc::KIND_MXF4_B16 ? 16 : 32;
  const int nt = osc::SPLIT_MAX_M;
  const uint64_t kb = fp8 ? (uint64_t)K : (uint64_t)K / 2;
  const int nslot4 = K / V / 4;
  const uint32_t aps = fp8 ? 1u : (V == 16 ? 4u : 2u);
  osc::SmallMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  int rc;
  {
    uint64_t d[2] = {kb, (uint64_t)N}, st[1] = {kb};
    uint32_t box[2] = {128, 128};
    if ((rc = make_map(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, QW, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
    uint64_t dx[2] = {kb, (uint64_t)M};
    uint32_t boxx[2] = {128, (uint32_t)nt};
    if ((rc = make_map(&maps.x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, QX, dx, st, boxx, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  }
  {
    // boxes of a whole scale chunk: SMALL_CHUNK_ATOMS atoms of one 128-row block
    uint64_t d[3] = {128, (uint64_t)nslot4, (uint64_t)((N + 127) / 128)}, st[2] = {512, (uint64_t)nslot4 * 512};
    uint32_t box[3] = {128, (uint32_t)osc::SMALL_CHUNK_ATOMS, 1};
    (void)aps;
    if ((rc = make_map(&maps.sw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, SW, d, st, box, CU_TENSOR_MAP_SWIZZLE_NONE))) return rc;
    uint64_t dx[3] = {128, (uint64_t)nslot4, 1};
    if ((rc = make_map(&maps.sx, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, SX, dx, st, box, CU_TENSOR_MAP_SWIZZLE_NONE))) return rc;
  }
  if (K_L > 0) {
    uint64_t d[2] = {(uint64_t)K_L, (uint64_t)N}, st[1] = {(uint64_t)K_L * 2};
    uint32_t box[2] = {64, 128};
    if ((rc = make_map(&maps.wl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, WL, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
    uint64_t db[2] = {(uint64_t)K_L, (uint64_t)M};
    uint32_t boxb[2] = {64, (uint32_t)nt};
    if ((rc = make_map(&maps.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, db, st, boxb, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  }
  osc::SmallParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = M; p.N = N; p.K = K; p.K_L = K_L;
  p.S = pl.S; p.n_tiles = pl.n_tiles; p.num_sms = ds->sms;
  p.Y = Y; p.Yf32 = Yf32; p.partial = workspace;
  p.status = ds->status;
  const int units = pl.n_tiles * pl.S;
  const int grid = units < ds->sms ? units : ds->sms;
  return launch_result(osc::launch_gemm_small(kind, maps, p, grid, stream));
}

// Shared launch path of the dense, fallback and grouped products.
int run_gemm(int kind, const uint8_t* QX, const uint8_t* SX, const uint16_t* B, const uint8_t* QW,
             const uint8_t* SW, const uint16_t* WL, int M, int N, int K, int K_L, int E,
             const int* mblock_expert, const int* kl, uint16_t* Y, float* Yf32, cudaStream_t stream,
             float* workspace = nullptr, size_t workspace_bytes = 0, bool preload = false) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  const bool fp8 = kind == osc::KIND_MXF8_B32;
  const int V = kind == osc::KIND_MXF4_B16 ? 16 : 32;
  int bn = g_tile_n.load();
  int cg = g_pair.load();
  const bool grouped = mblock_expert != nullptr;
  // few token rows with a workspace for split partials: the transposed split product, unless
  // a tile shape was forced (the tests use that to reach the general kernel there)
  if (!grouped && workspace != nullptr && M <= osc::SPLIT_MAX_M && bn == 0 && cg < 0) {
    const SmallPlan pl = small_plan(kind, M, N, K, K_L, ds->sms);
    if (pl.S > 1 && workspace_bytes >= pl.partial_bytes)
      return run_gemm_small(kind, QX, SX, B, QW, SW, WL, M, N, K, K_L, Y, Yf32, workspace, pl, ds, stream);
  }
  if (bn == 0) bn = (N >= 256 && (long long)((M + 127) / 128) * ((N + 255) / 256) >= ds->sms) ? 256 : 128;
  // the CTA pair needs 256-wide tiles, whole 256-row tiles of work and a per-128-row expert map
  // it cannot honour, so grouped calls stay on single CTAs
  // measured on the B200 (launches back to back, cold inputs): the 2-CTA pair is faster for
  // every 256-wide product with more than 128 rows - QKV 2048x6144x4096 29.6 vs 30.9 us,
  // 8192x6144x4096 94.4 vs 100.0 us, FFN 4096x24576x4096 193.4 vs 195.6 us; with 128 rows or
  // fewer half of its 256-row tile would be empty
  if (cg < 0) cg = (bn == 256 && !grouped && M > 128) ? 2 : 1;
  if (cg == 2 && (bn != 256 || grouped)) cg = 1;
  const int m_tiles = (M + 128 * cg - 1) / (128 * cg);

  osc::GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const uint64_t kb = fp8 ? (uint64_t)K : (uint64_t)K / 2;       // operand bytes per row
  const int nslot4 = K / V / 4;
  const int brows = bn / cg;
  {
    uint64_t d[2] = {kb, (uint64_t)M}, st[1] = {kb};
    uint32_t box[2] = {128, 128};
    if ((rc = make_map(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, QX, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  }
  {
    uint64_t d[3] = {kb, (uint64_t)N, (uint64_t)E}, st[2] = {kb, kb * (uint64_t)N};
    uint32_t box[3] = {128, (uint32_t)brows, 1};
    if ((rc = make_map(&maps.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, QW, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  }
  {
    // scale buffers as (128 words of an atom) x (atoms along K) x (128-row blocks)
    const uint64_t mblk = (uint64_t)((M + 127) / 128);
    uint64_t d[3] = {128, (uint64_t)nslot4, mblk}, st[2] = {512, (uint64_t)nslot4 * 512};
    uint32_t box[3] = {128, (uint32_t)(fp8 ? 1 : (V == 16 ? 4 : 2)), 1};
    if ((rc = make_map(&maps.sfa, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, SX, d, st, box, CU_TENSOR_MAP_SWIZZLE_NONE))) return rc;
    const uint64_t nblk = (uint64_t)((N + 127) / 128) * (uint64_t)E;
    uint64_t d2[3] = {128, (uint64_t)nslot4, nblk};
    uint32_t box2[3] = {128, box[1], (uint32_t)(bn / 128)};
    if ((rc = make_map(&maps.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, SW, d2, st, box2, CU_TENSOR_MAP_SWIZZLE_NONE))) return rc;
  }
  if (K_L > 0) {
    uint64_t d[2] = {(uint64_t)K_L, (uint64_t)M}, st[1] = {(uint64_t)K_L * 2};
    uint32_t box[2] = {64, 128};
    if ((rc = make_map(&maps.ca, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
    uint64_t d3[3] = {(uint64_t)K_L, (uint64_t)N, (uint64_t)E}, st3[2] = {(uint64_t)K_L * 2, (uint64_t)K_L * 2 * N};
    uint32_t box3[3] = {64, (uint32_t)brows, 1};
    if ((rc = make_map(&maps.cb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, WL, d3, st3, box3, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  }
  {
    uint64_t d[2] = {(uint64_t)N, (uint64_t)M}, st[1] = {(uint64_t)N * 2};
    uint32_t box[2] = {16, 32};
    if ((rc = make_map(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, d, st, box, CU_TENSOR_MAP_SWIZZLE_32B))) return rc;
  }
  osc::GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = M; p.N = N; p.K = K; p.K_L = K_L;
  p.SFA = SX; p.SFB = SW;
  p.nslot4 = nslot4;
  p.m_tiles = m_tiles;
  p.n_tiles = (N + bn - 1) / bn;
  p.Yf32 = Yf32;
  p.status = ds->status;
  p.num_groups = mblock_expert ? E : 0;
  p.mblock_expert = mblock_expert;
  p.group_kl = kl;
  p.preload = preload && mblock_expert == nullptr ? 1 : 0;
  const int tiles = p.m_tiles * p.n_tiles;
  const int units = ds->sms / cg;
  const int grid = (tiles < units ? tiles : units) * cg;
  return launch_result(osc::launch_gemm(kind, bn, cg, maps, p, grid, stream));
}

int check_linear_common(const void* QX, const void* SX, const void* QW, const void* SW, int M, int N, int K,
                        uint16_t* Y, float* Yf32) {
  if (!QX || !SX || !QW || !SW || !Y || M < 0 || N <= 0 || K <= 0) return OSC_ERR_ARG;
  if (!a16(QX) || !a16(SX) || !a16(QW) || !a16(SW) || !a16(Y) || (Yf32 && !a16(Yf32))) return OSC_ERR_ALIGN;
  if (K % 256 != 0 || N % 16 != 0) return OSC_ERR_ALIGN;
  return OSC_OK;
}

}  // namespace

extern "C" {

const char* osc_version(void) { return "osc-b200 0.1 (sm_100a)"; }

const char* osc_error_string(int code) {
  switch (code) {
    case OSC_OK: return "ok";
    case OSC_ERR_ARG: return "invalid argument (null pointer or unsupported size)";
    case OSC_ERR_ALIGN: return "alignment or divisibility requirement not met";
    case OSC_ERR_G: return "group size must be 16, 32 or 64";
    case OSC_ERR_CUDA: return "CUDA call failed (see osc_last_cuda_error)";
    case OSC_ERR_TIMEOUT: return "a kernel wait ran out of time";
    case OSC_ERR_TABLE: return "table entry out of range or more entries than K_L";
    case OSC_ERR_DEVICE: return "current device is not an sm_100 GPU";
    case OSC_ERR_SCRATCH: return "the split needs more partials than the fixed 16 MiB scratch holds";
    default: return "unknown error";
  }
}

int osc_last_cuda_error(void) { return t_last_cuda; }

size_t osc_scale_bytes(int rows, int K, int G) {
  if (rows < 0 || K <= 0) return 0;
  int V;
  if (G == 0) V = 32;
  else if (valid_g(G)) V = (G == 16) ? 16 : 32;
  else return 0;
  if (K % (4 * V) != 0) return 0;
  return (size_t)((rows + 127) / 128) * (size_t)(K / V / 4) * 512u;
}

int osc_table_kl(const int8_t* L_host, int Kg) {
  if (!L_host || Kg < 0) return OSC_ERR_ARG;
  int c = 0;
  for (int k = 0; k < Kg; ++k) c += (L_host[k] >= 0);
  return (c + 15) / 16 * 16;
}

int osc_set_tile_n(int bn) {
  if (bn != 0 && bn != 128 && bn != 256) return OSC_ERR_ARG;
  return g_tile_n.exchange(bn);
}

int osc_set_cta_pair(int mode) {
  if (mode != -1 && mode != 1 && mode != 2) return OSC_ERR_ARG;
  return g_pair.exchange(mode);
}

int osc_build_table_multi(const uint16_t* Xcal, int S, int K, int G, float alpha, int min_hits, int R, int8_t* L,
                          osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (!Xcal || !L || S < 0 || K <= 0 || K % G != 0 || R < 1 || R > osc::MAX_R) return OSC_ERR_ARG;
  if (!a16(Xcal)) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  osc::TableParams p{Xcal, S, K, G, alpha, min_hits, R, L};
  return launch_result(osc::launch_build_table(p, ds->sms, (cudaStream_t)stream));
}

int osc_build_table(const uint16_t* Xcal, int S, int K, int G, float alpha, int min_hits, int8_t* L,
                    osc_stream_t stream) {
  return osc_build_table_multi(Xcal, S, K, G, alpha, min_hits, 1, L, stream);
}

int osc_density(const uint16_t* X, int S, int K, int G, float alpha, const int8_t* L, int* n_hit, int* n_total,
                osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (!X || !L || !n_hit || !n_total || S < 0 || K <= 0 || K % G != 0) return OSC_ERR_ARG;
  if (!a16(X)) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  osc::DensityParams p{X, S, K, G, alpha, L, n_hit, n_total, ds->status};
  return launch_result(osc::launch_density(p, (cudaStream_t)stream));
}

namespace {
// The tier of §2.3 for a clustering density C (NaN: no events, nothing escapes the table).
int tier_of(double c) {
  if (std::isnan(c)) return OSC_TIER_HIGH;
  return c > 0.60 ? OSC_TIER_HIGH : (c >= 0.35 ? OSC_TIER_MID : OSC_TIER_FP8);
}
}  // namespace

int osc_select_group_size(const double* c_bar, int* tier) {
  if (!c_bar) return OSC_ERR_ARG;
  static const int kG[3] = {16, 32, 64};
  int best = 0;
  for (int i = 0; i < 3; ++i)
    if (tier_of(c_bar[i]) == OSC_TIER_HIGH) best = kG[i];
  if (best != 0) {
    if (tier) *tier = OSC_TIER_HIGH;
    return best;
  }
  const int t = tier_of(c_bar[1]);
  if (tier) *tier = t;
  return t == OSC_TIER_FP8 ? 0 : 32;
}

int osc_select_tier(const int* n_hit, const int* n_total, int Kg, double* c_bar) {
  if (Kg < 0 || (Kg > 0 && (!n_hit || !n_total))) return OSC_ERR_ARG;
  double sum = 0.0;
  int groups = 0;
  for (int k = 0; k < Kg; ++k) {
    if (n_hit[k] < 0 || n_total[k] < 0 || n_hit[k] > n_total[k]) return OSC_ERR_ARG;
    if (n_total[k] > 0) {
      sum += (double)n_hit[k] / (double)n_total[k];
      ++groups;
    }
  }
  if (groups == 0) {
    if (c_bar) *c_bar = std::nan("");
    return OSC_TIER_HIGH;
  }
  const double c = sum / groups;
  if (c_bar) *c_bar = c;
  return tier_of(c);
}

int osc_quantize(const uint16_t* X, int M, int K, int G, const int8_t* L, int R, int K_L, uint8_t* QX, uint8_t* SX,
                 uint16_t* B, osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (R < 1 || R > osc::MAX_R) return OSC_ERR_ARG;
  if (M == 0 && K > 0 && K_L >= 0) return OSC_OK;          // nothing to read or write
  if (!X || !QX || !SX || M < 0 || K <= 0 || K_L < 0) return OSC_ERR_ARG;
  if ((long long)(M + 127) * (K / 32) >= (1LL << 31)) return OSC_ERR_ARG;
  if (L == nullptr && K_L != 0) return OSC_ERR_ARG;
  if (L != nullptr && K_L > 0 && !B) return OSC_ERR_ARG;
  if (K_L > 32767 || (L != nullptr && (long long)(K / G) * R > osc::MAX_TAB)) return OSC_ERR_ARG;
  if (!a16(X) || !a16(QX) || !a16(SX) || (B && !a16(B))) return OSC_ERR_ALIGN;
  if (K % 256 != 0 || K_L % 16 != 0) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  if (M == 0) return OSC_OK;
  osc::QuantParams p{X, M, K, G, K / G, L, R, K_L, QX, SX, B, ds->status};
  CUtensorMap tm;
  if ((rc = make_block_map(&tm, X, M, K))) return rc;
  return launch_result(osc::launch_quantize(tm, p, false, ds->sms, (cudaStream_t)stream));
}

int osc_rmsnorm_quantize(const uint16_t* X, const uint16_t* gamma, float eps, int M, int K, int G, const int8_t* L,
                         int R, int K_L, uint8_t* QX, uint8_t* SX, uint16_t* B, osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (R < 1 || R > osc::MAX_R) return OSC_ERR_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return OSC_ERR_ARG;
  if (M == 0 && K > 0 && K_L >= 0) return OSC_OK;          // nothing to read or write
  if (!X || !gamma || !QX || !SX || M < 0 || K <= 0 || K_L < 0) return OSC_ERR_ARG;
  if (K > osc::NQ_MAX_K) return OSC_ERR_ARG;
  if ((long long)(M + 127) * (K / 32) >= (1LL << 31)) return OSC_ERR_ARG;
  if (L == nullptr && K_L != 0) return OSC_ERR_ARG;
  if (L != nullptr && K_L > 0 && !B) return OSC_ERR_ARG;
  if (K_L > 32767) return OSC_ERR_ARG;
  if (!a16(X) || !a16(gamma) || !a16(QX) || !a16(SX) || (B && !a16(B))) return OSC_ERR_ALIGN;
  if (K % 256 != 0 || K_L % 16 != 0) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  osc::NormQuantParams p{X, gamma, eps, M, K, G, K / G, L, R, K_L, QX, SX, B, ds->status};
  CUtensorMap tm;
  if ((rc = make_row_map(&tm, X, M, K))) return rc;
  return launch_result(osc::launch_rmsnorm_quantize(tm, p, ds->sms, (cudaStream_t)stream));
}

int osc_prepare_weight(const uint16_t* W, int N, int K, int G, const int8_t* L, int R, int K_L, uint8_t* QW,
                       uint8_t* SW, uint16_t* WL, osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (R < 1 || R > osc::MAX_R) return OSC_ERR_ARG;
  if (!W || !QW || !SW || N < 0 || K <= 0 || K_L < 0) return OSC_ERR_ARG;
  if ((long long)(N + 127) * (K / 32) >= (1LL << 31)) return OSC_ERR_ARG;
  if (K_L > 0 && (!L || !WL)) return OSC_ERR_ARG;
  if (!a16(W) || !a16(QW) || !a16(SW) || (WL && !a16(WL))) return OSC_ERR_ALIGN;
  if (K % 256 != 0 || K_L % 16 != 0) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  if (N == 0) return OSC_OK;
  osc::QuantParams p{W, N, K, G, K / G, nullptr, 1, 0, QW, SW, nullptr, ds->status};
  CUtensorMap tm;
  if ((rc = make_block_map(&tm, W, N, K))) return rc;
  cudaError_t e = osc::launch_quantize(tm, p, false, ds->sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail_cuda(e);
  return launch_result(osc::launch_gather_wl(W, N, K, G, L, R, K_L, WL, ds->status, ds->sms, (cudaStream_t)stream));
}

int osc_linear(const uint8_t* QX, const uint8_t* SX, const uint16_t* B, const uint8_t* QW, const uint8_t* SW,
               const uint16_t* WL, int M, int N, int K, int G, int K_L, uint16_t* Y, float* Yf32,
               osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (M == 0 && N > 0 && K > 0 && K_L >= 0) return OSC_OK;  // nothing to read or write
  int rc = check_linear_common(QX, SX, QW, SW, M, N, K, Y, Yf32);
  if (rc != OSC_OK) return rc;
  if (K_L < 0 || K_L % 16 != 0) return K_L < 0 ? OSC_ERR_ARG : OSC_ERR_ALIGN;
  if (K_L > 0 && (!B || !WL)) return OSC_ERR_ARG;
  if (K_L > 0 && (!a16(B) || !a16(WL))) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != OSC_OK) return rc;
  const int kind = G == 16 ? osc::KIND_MXF4_B16 : osc::KIND_MXF4_B32;
  return run_gemm(kind, QX, SX, B, QW, SW, WL, M, N, K, K_L, 1, nullptr, nullptr, Y, Yf32, (cudaStream_t)stream);
}

int osc_quantize_linear(const uint16_t* X, int M, int K, int G, const int8_t* L, int R, int K_L, uint8_t* QX,
                        uint8_t* SX, uint16_t* B, const uint8_t* QW, const uint8_t* SW, const uint16_t* WL, int N,
                        uint16_t* Y, float* Yf32, float* workspace, size_t workspace_bytes, osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (R < 1 || R > osc::MAX_R) return OSC_ERR_ARG;
  if (M == 0 && N > 0 && K > 0 && K_L >= 0) return OSC_OK;  // nothing to read or write
  // every argument of both steps is checked before anything is launched
  if (!X || M < 0 || K_L < 0) return OSC_ERR_ARG;
  if ((long long)(M + 127) * (K / 32) >= (1LL << 31)) return OSC_ERR_ARG;
  if (L == nullptr && K_L != 0) return OSC_ERR_ARG;
  if (K_L > 0 && (!B || !WL)) return OSC_ERR_ARG;
  if (K_L > 32767 || (L != nullptr && (long long)(K / G) * R > osc::MAX_TAB)) return OSC_ERR_ARG;
  int rc = check_linear_common(QX, SX, QW, SW, M, N, K, Y, Yf32);
  if (rc != OSC_OK) return rc;
  if (!a16(X) || (B && !a16(B)) || (WL && !a16(WL))) return OSC_ERR_ALIGN;
  if (K_L % 16 != 0) return OSC_ERR_ALIGN;
  if (workspace_bytes > 0 && !workspace) return OSC_ERR_ARG;
  if (workspace && !a16(workspace)) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != OSC_OK) return rc;
  osc::QuantParams qp{X, M, K, G, K / G, L, R, K_L, QX, SX, B, ds->status};
  CUtensorMap tm;
  if ((rc = make_block_map(&tm, X, M, K))) return rc;
  if ((rc = launch_result(osc::launch_quantize(tm, qp, false, ds->sms, (cudaStream_t)stream))) != OSC_OK) return rc;
  const int kind = G == 16 ? osc::KIND_MXF4_B16 : osc::KIND_MXF4_B32;
  return run_gemm(kind, QX, SX, B, QW, SW, WL, M, N, K, K_L, 1, nullptr, nullptr, Y, Yf32, (cudaStream_t)stream,
                  workspace, workspace_bytes, true);
}

int osc_rmsnorm_quantize_linear(const uint16_t* X, const uint16_t* gamma, float eps, int M, int K, int G,
                                const int8_t* L, int R, int K_L, uint8_t* QX, uint8_t* SX, uint16_t* B,
                                const uint8_t* QW, const uint8_t* SW, const uint16_t* WL, int N, uint16_t* Y,
                                float* Yf32, osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (R < 1 || R > osc::MAX_R) return OSC_ERR_ARG;
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return OSC_ERR_ARG;
  if (M == 0 && N > 0 && K > 0 && K_L >= 0) return OSC_OK;  // nothing to read or write
  // every argument of both steps is checked before anything is launched
  if (!X || !gamma || M < 0 || K_L < 0) return OSC_ERR_ARG;
  if (K > osc::NQ_MAX_K) return OSC_ERR_ARG;
  if ((long long)(M + 127) * (K / 32) >= (1LL << 31)) return OSC_ERR_ARG;
  if (L == nullptr && K_L != 0) return OSC_ERR_ARG;
  if (K_L > 0 && (!B || !WL)) return OSC_ERR_ARG;
  if (K_L > 32767) return OSC_ERR_ARG;
  int rc = check_linear_common(QX, SX, QW, SW, M, N, K, Y, Yf32);
  if (rc != OSC_OK) return rc;
  if (!a16(X) || !a16(gamma) || (B && !a16(B)) || (WL && !a16(WL))) return OSC_ERR_ALIGN;
  if (K_L % 16 != 0) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != OSC_OK) return rc;
  osc::NormQuantParams qp{X, gamma, eps, M, K, G, K / G, L, R, K_L, QX, SX, B, ds->status};
  CUtensorMap tm;
  if ((rc = make_row_map(&tm, X, M, K))) return rc;
  if ((rc = launch_result(osc::launch_rmsnorm_quantize(tm, qp, ds->sms, (cudaStream_t)stream))) != OSC_OK) return rc;
  const int kind = G == 16 ? osc::KIND_MXF4_B16 : osc::KIND_MXF4_B32;
  return run_gemm(kind, QX, SX, B, QW, SW, WL, M, N, K, K_L, 1, nullptr, nullptr, Y, Yf32, (cudaStream_t)stream,
                  nullptr, 0, true);
}

size_t osc_linear_workspace_bytes(int M, int N, int K, int K_L) {
  if (M <= 0 || M > osc::SPLIT_MAX_M || N <= 0 || K <= 0 || K_L < 0 || K % 256 != 0 || N % 16 != 0 || K_L % 16 != 0)
    return 0;
  DeviceState* ds = nullptr;
  if (device_state(&ds) != OSC_OK) return 0;
  return small_plan(osc::KIND_MXF4_B32, M, N, K, K_L, ds->sms).partial_bytes;
}

int osc_linear_splitk(const uint8_t* QX, const uint8_t* SX, const uint16_t* B, const uint8_t* QW, const uint8_t* SW,
                      const uint16_t* WL, int M, int N, int K, int G, int K_L, uint16_t* Y, float* Yf32,
                      float* workspace, size_t workspace_bytes, osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (M == 0 && N > 0 && K > 0 && K_L >= 0) return OSC_OK;  // nothing to read or write
  int rc = check_linear_common(QX, SX, QW, SW, M, N, K, Y, Yf32);
  if (rc != OSC_OK) return rc;
  if (K_L < 0 || K_L % 16 != 0) return K_L < 0 ? OSC_ERR_ARG : OSC_ERR_ALIGN;
  if (K_L > 0 && (!B || !WL)) return OSC_ERR_ARG;
  if (K_L > 0 && (!a16(B) || !a16(WL))) return OSC_ERR_ALIGN;
  if (workspace_bytes > 0 && !workspace) return OSC_ERR_ARG;
  if (workspace && !a16(workspace)) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != OSC_OK) return rc;
  const int kind = G == 16 ? osc::KIND_MXF4_B16 : osc::KIND_MXF4_B32;
  return run_gemm(kind, QX, SX, B, QW, SW, WL, M, N, K, K_L, 1, nullptr, nullptr, Y, Yf32, (cudaStream_t)stream,
                  workspace, workspace_bytes);
}

int osc_quantize_fp8(const uint16_t* X, int M, int K, uint8_t* QX8, uint8_t* SX, osc_stream_t stream) {
  if (M == 0 && K > 0) return OSC_OK;                       // nothing to read or write
  if (!X || !QX8 || !SX || M < 0 || K <= 0) return OSC_ERR_ARG;
  if ((long long)(M + 127) * (K / 32) >= (1LL << 31)) return OSC_ERR_ARG;
  if (!a16(X) || !a16(QX8) || !a16(SX)) return OSC_ERR_ALIGN;
  if (K % 256 != 0) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  if (M == 0) return OSC_OK;
  osc::QuantParams p{X, M, K, 32, K / 32, nullptr, 1, 0, QX8, SX, nullptr, ds->status};
  CUtensorMap tm;
  if ((rc = make_block_map(&tm, X, M, K))) return rc;
  return launch_result(osc::launch_quantize(tm, p, true, ds->sms, (cudaStream_t)stream));
}

int osc_linear_fp8_fallback(const uint8_t* QX8, const uint8_t* SX, const uint8_t* QW8, const uint8_t* SW, int M,
                            int N, int K, uint16_t* Y, float* Yf32, osc_stream_t stream) {
  if (M == 0 && N > 0 && K > 0) return OSC_OK;              // nothing to read or write
  int rc = check_linear_common(QX8, SX, QW8, SW, M, N, K, Y, Yf32);
  if (rc != OSC_OK) return rc;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != OSC_OK) return rc;
  if (M == 0) return OSC_OK;
  return run_gemm(osc::KIND_MXF8_B32, QX8, SX, nullptr, QW8, SW, nullptr, M, N, K, 0, 1, nullptr, nullptr, Y, Yf32,
                  (cudaStream_t)stream);
}

int osc_grouped_plan(const int* counts, int E, int* off, int* poff, int* mblock_expert, int mblock_capacity) {
  if (!counts || !off || !poff || E <= 0 || mblock_capacity < 0) return OSC_ERR_ARG;
  long long o = 0, po = 0;
  for (int e = 0; e < E; ++e) {
    if (counts[e] < 0) return OSC_ERR_ARG;
    off[e] = (int)o;
    poff[e] = (int)po;
    o += counts[e];
    po += (counts[e] + 127) / 128 * 128;
    if (po > 0x7FFFFF80LL) return OSC_ERR_ARG;
  }
  off[E] = (int)o;
  poff[E] = (int)po;
  if (mblock_expert) {
    if (po / 128 > mblock_capacity) return OSC_ERR_ARG;
    for (int e = 0; e < E; ++e)
      for (int b = poff[e] / 128; b < poff[e + 1] / 128; ++b) mblock_expert[b] = e;
  }
  return (int)po;
}

int osc_quantize_grouped(const uint16_t* X, int T, int E, const int* off, const int* poff, const int* mblock_expert,
                         int Mp, int K, int G, const int8_t* L, int R, int K_L, uint8_t* QX, uint8_t* SX, uint16_t* B,
                         osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (R < 1 || R > osc::MAX_R) return OSC_ERR_ARG;
  if (!X || !off || !poff || !mblock_expert || !L || !QX || !SX || E <= 0 || Mp < 0 || K <= 0 || K_L < 0)
    return OSC_ERR_ARG;
  if (T < 0 || T > Mp) return OSC_ERR_ARG;
  if (K_L > 0 && !B) return OSC_ERR_ARG;
  if (K_L > 32767) return OSC_ERR_ARG;
  if ((long long)(Mp + 127) * (K / 32) >= (1LL << 31)) return OSC_ERR_ARG;
  if (!a16(X) || !a16(QX) || !a16(SX) || (B && !a16(B))) return OSC_ERR_ALIGN;
  if (K % 256 != 0 || K_L % 16 != 0 || Mp % 128 != 0) return OSC_ERR_ALIGN;
  if (osc::grouped_quant_smem(E, K / G, R) > (size_t)osc::GROUPED_QUANT_SMEM_MAX) return OSC_ERR_ARG;   // E x K/G x R entries
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  if (Mp == 0) return OSC_OK;
  osc::GroupedQuantParams p{X, off, poff, mblock_expert, E, Mp, K, G, K / G, L, R, K_L, QX, SX, B, ds->status};
  if (T > 0 && osc::grouped_tma_smem(E, K / G, R) <= (size_t)osc::GROUPED_TMA_SMEM_MAX) {
    CUtensorMap tm;
    if ((rc = make_block_map(&tm, X, T, K))) return rc;
    return launch_result(osc::launch_quantize_grouped_tma(tm, p, T, ds->sms, (cudaStream_t)stream));
  }
  return launch_result(osc::launch_quantize_grouped(p, ds->sms, (cudaStream_t)stream));
}

int osc_linear_grouped(const uint8_t* QX, const uint8_t* SX, const uint16_t* B, const uint8_t* QW, const uint8_t* SW,
                       const uint16_t* WL, const int* mblock_expert, const int* kl, int E, int Mp, int N, int K,
                       int G, int K_L, uint16_t* Y, float* Yf32, osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  int rc = check_linear_common(QX, SX, QW, SW, Mp, N, K, Y, Yf32);
  if (rc != OSC_OK) return rc;
  if (!mblock_expert || E <= 0) return OSC_ERR_ARG;
  if (Mp % 128 != 0) return OSC_ERR_ALIGN;
  if (K_L < 0 || K_L % 16 != 0) return K_L < 0 ? OSC_ERR_ARG : OSC_ERR_ALIGN;
  if (K_L > 0 && (!B || !WL)) return OSC_ERR_ARG;
  if (K_L > 0 && (!a16(B) || !a16(WL))) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != OSC_OK) return rc;
  if (Mp == 0) return OSC_OK;
  const int kind = G == 16 ? osc::KIND_MXF4_B16 : osc::KIND_MXF4_B32;
  return run_gemm(kind, QX, SX, B, QW, SW, WL, Mp, N, K, K_L, E, mblock_expert, K_L > 0 ? kl : nullptr, Y, Yf32,
                  (cudaStream_t)stream);
}

int osc_selftest_timeout(int limit_us, osc_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return OSC_ERR_ARG;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  return launch_result(osc::launch_selftest_wait(ds->status, 1000ull * (unsigned long long)limit_us,
                                                 (cudaStream_t)stream));
}

int osc_status(int* raw, osc_stream_t stream) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != OSC_OK) return rc;
  int v = 0;
  std::lock_guard<std::mutex> lock(ds->status_mu);
  status_take_kernel<<<1, 1, 0, (cudaStream_t)stream>>>();
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpyAsync(&v, ds->taken, sizeof(int), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return fail_cuda(e);
  if (raw) *raw = v;
  if (v == osc::DEV_TIMEOUT) return OSC_ERR_TIMEOUT;
  if (v == osc::DEV_BAD_TABLE) return OSC_ERR_TABLE;
  return OSC_OK;
}

}  // extern "C"

// ---- the allocation-free split product ------------------------------------------------------
// Some callers cannot allocate device memory (an engine plugin that is handed only its inputs
// and outputs, a serving loop that forbids allocation after start-up), so they cannot give
// osc_linear_splitk a workspace. For them the partials live in this fixed, file-scope device
// buffer. In host code the name g_noalloc_scratch is only a host-side stand-in; the kernels get
// the device address that cudaGetSymbolAddress returns, looked up once per device.
namespace {

static __device__ __align__(256) float g_noalloc_scratch[OSC_NOALLOC_SCRATCH_BYTES / sizeof(float)];

struct ScratchAddr {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  float* ptr = nullptr;
};

// Device address of the buffer on the current device (looked up on the first call for it).
int noalloc_scratch(float** out) {
  static ScratchAddr addr[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return OSC_ERR_DEVICE;
  ScratchAddr& a = addr[dev];
  std::call_once(a.once, [&] {
    void* p = nullptr;
    a.err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    a.ptr = static_cast<float*>(p);
  });
  if (a.err != cudaSuccess) return fail_cuda(a.err);
  *out = a.ptr;
  return OSC_OK;
}

}  // namespace

extern "C" int osc_linear_splitk_noalloc(const uint8_t* QX, const uint8_t* SX, const uint16_t* B, const uint8_t* QW,
                                         const uint8_t* SW, const uint16_t* WL, int M, int N, int K, int G, int K_L,
                                         uint16_t* Y, float* Yf32, osc_stream_t stream) {
  if (!valid_g(G)) return OSC_ERR_G;
  if (M == 0 && N > 0 && K > 0 && K_L >= 0) return OSC_OK;  // nothing to read or write
  int rc = check_linear_common(QX, SX, QW, SW, M, N, K, Y, Yf32);
  if (rc != OSC_OK) return rc;
  if (K_L < 0 || K_L % 16 != 0) return K_L < 0 ? OSC_ERR_ARG : OSC_ERR_ALIGN;
  if (K_L > 0 && (!B || !WL)) return OSC_ERR_ARG;
  if (K_L > 0 && (!a16(B) || !a16(WL))) return OSC_ERR_ALIGN;
  DeviceState* ds = nullptr;
  if ((rc = device_state(&ds)) != OSC_OK) return rc;
  const int kind = G == 16 ? osc::KIND_MXF4_B16 : osc::KIND_MXF4_B32;
  if (small_plan(kind, M, N, K, K_L, ds->sms).partial_bytes > (size_t)OSC_NOALLOC_SCRATCH_BYTES)
    return OSC_ERR_SCRATCH;
  float* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch)) != OSC_OK) return rc;
  return run_gemm(kind, QX, SX, B, QW, SW, WL, M, N, K, K_L, 1, nullptr, nullptr, Y, Yf32, (cudaStream_t)stream,
                  scratch, (size_t)OSC_NOALLOC_SCRATCH_BYTES);
}
