// fp8gemm_api.cu -- host side of the C ABI declared in include/fp8gemm.h:
// argument validation, TMA tensor-map encoding, kernel selection and launch.
// Every GEMM call is one kernel launch on the caller's stream; nothing here
// allocates after fg_init, reads device memory or synchronises.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fp8_cast_kernels.cuh"
#include "fp8_gemm_kernels.cuh"
#include "fp8gemm.h"
#include "fp8gemm_jit.h"
#include "fg_jit_sources.inc"  // the kernel headers, embedded at build time (build.py)

namespace {

using fg::kBlockK;
using fg::kBlockM;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;
constexpr unsigned kKnownFlags = FG_FLAG_STATIC_B;
constexpr int kMaxSwapMP = 128;
constexpr int kCounterCapacity = 1 << 16;  // n-tiles of 128 rows: N <= 8,388,608 on the stream-K path

struct DeviceState {
  bool ready = false;
  int sms = 0;
  int* status = nullptr;
  float* ws = nullptr;   // split-K partial tiles
  int* counters = nullptr;
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;
std::atomic<int> g_dense_path{0};
std::atomic<int> g_debug_stall{0};
// Tiled kernel: the last partial wave of tiles is split in K over all CTAs (stream-K tail) when
// its cost on the busiest CTA -- its units, this many K blocks for publishing partial tiles (a
// CTA may publish twice, about 3.4 us = 7 K blocks each, measured) and 2.4 K blocks per piece
// summed -- is at most the tile it replaces; 0: whenever the last wave is partial; negative: never.
#ifndef FG_TILED_SK_OVERHEAD
#define FG_TILED_SK_OVERHEAD 18
#endif
std::atomic<int> g_tiled_sk{FG_TILED_SK_OVERHEAD};
// Small-M kernel schedule: 0 automatic, -1 never a cluster split, 2/4/8 the cluster split with
// that many CTAs per tile wherever it is possible.
std::atomic<int> g_swap_schedule{0};
std::atomic<uint64_t> g_launches{0};

// tiled kernel configuration: 128 x 192 output tiles, 4-stage ring (overridable when building)
#ifndef FG_TILED_BN
#define FG_TILED_BN 192
#endif
#ifndef FG_TILED_STAGES
#define FG_TILED_STAGES 4
#endif
#ifndef FG_TILED_GROUP_MB
#define FG_TILED_GROUP_MB 24  // L2 budget (MB) for the A rows of one group of m-blocks
#endif
constexpr int kTiledBN = FG_TILED_BN;
#ifndef FG_TILED_BN_MAX
#define FG_TILED_BN_MAX 256  // widest tile of any tiled-kernel instance (sizes the split-K partials)
#endif
static_assert(kTiledBN <= FG_TILED_BN_MAX, "tile wider than the workspace allows");
constexpr int kTiledStages = FG_TILED_STAGES;
// CTA-pair kernel: 256 x 192 tiles per pair, each CTA's stage = 128 A rows + 96 B rows
#ifndef FG_PAIR_BN
#define FG_PAIR_BN 192
#endif
#ifndef FG_PAIR_STAGES
#define FG_PAIR_STAGES 5
#endif
constexpr int kPairBN = FG_PAIR_BN;
constexpr int kPairStages = FG_PAIR_STAGES;

// tile width of the tiled and pair kernels: 0 automatic, else forced (fg_set_tile_n)
std::atomic<int> g_tile_n{0};
// tile walk of the tiled family: 0 automatic, 1 groups of m-blocks (m fastest), 2 n fastest
std::atomic<int> g_tile_order{0};

// Tile walk (TiledParams::group_m): m-blocks in groups of group_m, m-block fastest inside a group;
// group_m = 1 walks every n-block of an m-block before the next m-block (n fastest).  When one
// group's (or the whole) B is small enough to stay in L2 (<= 40 MB), n fastest reads A once and B
// once: the ~148 tiles in flight cover a few m-blocks and every n-block, so B stays resident while
// A streams -- and in the grouped layouts consecutive m-blocks share an expert.  Larger B streams
// through, with A in groups whose rows take at most FG_TILED_GROUP_MB of L2.  rows: rows per
// m-block (128, or 256 for the CTA pair); mb_all: m-blocks in the walk.
int tile_group_m(long long rows, int N, int K, long long mb_all, int* b_resident) {
  constexpr long long kResidentB = 40ll << 20;
  const int order = g_tile_order.load(std::memory_order_relaxed);
  const long long b_bytes = static_cast<long long>(N) * K;
  *b_resident = (order == 2 || (order == 0 && b_bytes <= kResidentB)) ? 1 : 0;
  if (*b_resident) return 1;
  long long gm = (static_cast<long long>(FG_TILED_GROUP_MB) << 20) / (rows * K);
  if (gm < 1) gm = 1;
  if (gm > mb_all) gm = mb_all;
  return static_cast<int>(gm);
}

template <int BN>
constexpr int tiled_stages() {
  return BN == 128 ? 5 : (BN == 192 ? kTiledStages : 3);
}
template <int BN, int KPS = 1>
constexpr int pair_stages() {
  return KPS == 1 ? (BN == 192 ? kPairStages : 4) : 2;
}

template <int BN, int STAGES>
constexpr size_t tiled_smem_bytes() {
  return 1024 /*alignment slack*/ + static_cast<size_t>(STAGES) * (kBlockM + BN) * kBlockK +
         static_cast<size_t>(fg::kPromoWarps) * (BN / 64) * fg::kStoreBoxBytes /*output staging*/ +
         2 * (fg::kSaChunk * kBlockM + 2 * fg::kSaChunk) * 4 /*scale chunks*/ + 256 /*barriers*/ +
         4 * (fg::kMaskedMaxGroups + 1) /*masked prefix*/;
}
static_assert(tiled_smem_bytes<kTiledBN, kTiledStages>() <= 227 * 1024, "tiled kernel shared memory");
static_assert(tiled_smem_bytes<128, tiled_stages<128>()>() <= 227 * 1024, "tiled kernel shared memory");
static_assert(tiled_smem_bytes<256, tiled_stages<256>()>() <= 227 * 1024, "tiled kernel shared memory");

template <int BN, int STAGES, int KPS = 1>
constexpr size_t pair_smem_bytes() {
  return 1024 + static_cast<size_t>(STAGES) * KPS * (kBlockM + BN / 2) * kBlockK +
         static_cast<size_t>(fg::kPromoWarps) * (BN / 64) * fg::kStoreBoxBytes +
         2 * (fg::kSaChunk * kBlockM + 2 * fg::kSaChunk) * 4 + 256 + 4 * (fg::kMaskedMaxGroups + 1);
}
static_assert(pair_smem_bytes<kPairBN, kPairStages>() <= 227 * 1024, "pair kernel shared memory");
static_assert(pair_smem_bytes<256, pair_stages<256>()>() <= 227 * 1024, "pair kernel shared memory");
static_assert(pair_smem_bytes<256, pair_stages<256, 2>(), 2>() <= 227 * 1024, "pair kernel shared memory");
static_assert(pair_smem_bytes<192, pair_stages<192, 2>(), 2>() <= 227 * 1024, "pair kernel shared memory");

// Ring stages of the small-M kernel by MP and K blocks per stage (KPS): about 192 KB of ring.
template <int MP, int KPS = 1>
constexpr int swap_stages() {
  return KPS == 1 ? (MP == 128 ? 5 : (MP == 64 ? 8 : 10)) : (MP == 128 ? 2 : (MP == 64 ? 4 : 5));
}

template <int MP, int STAGES, int KPS = 1>
constexpr size_t swap_smem_bytes() {
  return 1024 + static_cast<size_t>(STAGES) * KPS * (kBlockM + MP) * kBlockK + MP * kBlockM * 2 /*C staging*/ +
         fg::kSwapScaleBytes /*combined scales*/ + fg::kSwapBarrierBytes;
}
static_assert(swap_smem_bytes<32, swap_stages<32, 2>(), 2>() <= 227 * 1024, "swap kernel shared memory");
static_assert(swap_smem_bytes<64, swap_stages<64, 2>(), 2>() <= 227 * 1024, "swap kernel shared memory");
static_assert(swap_smem_bytes<128, swap_stages<128, 2>(), 2>() <= 227 * 1024, "swap kernel shared memory");

// K blocks per stage of the small-M kernel: 0 automatic (2 when K is a multiple of 128, else 1),
// or 1 / 2 forced (2 only where K allows it; fg_set_stage_kblocks)
std::atomic<int> g_stage_kb{0};
// promotion warpgroups of the 256-wide CTA-pair kernel (2 or 4; fg_set_pair_promotion)
std::atomic<int> g_pair_pw{2};

// K blocks per stage of the CTA-pair kernel: 2 when K is a multiple of 128 with at least two K
// blocks, unless fg_set_stage_kblocks forces 1.
int pair_kps_for(int K) {
  const int f = g_stage_kb.load(std::memory_order_relaxed);
  return (K % 128 == 0 && K >= 256 && f != 1) ? 2 : 1;
}

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// What one GEMM launch uses besides its operands: the SM count, the status word, and the split-K
// workspace (partial tiles + per-tile counters) -- the library's own (fg_init) or the caller's.
struct Ctx {
  int sms = 0;
  int* status = nullptr;
  float* ws = nullptr;
  int* counters = nullptr;
};

// Split-K workspace layout (library-owned and caller-owned alike): two partial tiles per SM of
// 128 x max(swap MP, tiled BN) fp32, then kCounterCapacity int counters (zero between launches).
size_t workspace_partial_bytes(int sms) {
  return static_cast<size_t>(2) * sms * kBlockM * (kMaxSwapMP > FG_TILED_BN_MAX ? kMaxSwapMP : FG_TILED_BN_MAX) *
         sizeof(float);
}
size_t workspace_bytes_for(int sms) { return workspace_partial_bytes(sms) + kCounterCapacity * sizeof(int); }

Ctx ctx_of(const DeviceState* st) {
  Ctx c;
  c.sms = st->sms;
  c.status = st->status;
  c.ws = st->ws;
  c.counters = st->counters;
  return c;
}

DeviceState* state_for_current(fg_status* err) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices || !g_dev[dev].ready) {
    *err = FG_ERR_NOT_INITIALIZED;
    return nullptr;
  }
  return &g_dev[dev];
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// 3-D map over e4m3 codes: dims {K, rows, groups}, box {128, box_rows, 1}, 128-byte swizzle,
// out-of-bounds elements read as zero.
bool encode_fp8_map(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint64_t groups,
                    uint32_t box_rows) {
  cuuint64_t dims[3] = {K, rows, groups};
  cuuint64_t strides[2] = {K, K * rows};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kBlockK), box_rows, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 output map for TMA stores: dims {N, rows[, groups]}, box {32, 32[, 1]}, 64-byte swizzle
// (the staging layout of the tiled kernel's epilogue).
bool encode_bf16_store_map(CUtensorMap* map, void* base, uint64_t N, uint64_t rows, uint64_t groups, bool three_d) {
  cuuint64_t dims[3] = {N, rows, groups};
  cuuint64_t strides[2] = {N * 2, N * 2 * rows};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, three_d ? 3 : 2, base, dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view of a K-major e4m3 matrix [rows, K] (K a multiple of 128) as {128 bytes of a K block,
// rows, K blocks} with strides {K, 128}: a box {128, box_rows, kps} is kps consecutive K blocks of
// box_rows rows, laid out in shared memory as kps tiles of box_rows x 128 bytes one after the other
// (each 128-byte swizzled like a 2-D copy of it).
bool encode_fp8_map_kblocks(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows,
                            uint32_t kps) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kBlockK), rows, K / kBlockK};
  cuuint64_t strides[2] = {K, static_cast<cuuint64_t>(kBlockK)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kBlockK), box_rows, kps};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D view of a grouped K-major e4m3 tensor [groups, rows, K] (K a multiple of 128) as {128 bytes,
// rows, K blocks, groups}: a box {128, box_rows, kps, 1} is kps consecutive K blocks of box_rows
// rows of one group, laid out as kps swizzled tiles one after the other.
bool encode_fp8_map_kblocks_grouped(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint64_t groups,
                                    uint32_t box_rows, uint32_t kps) {
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(kBlockK), rows, K / kBlockK, groups};
  cuuint64_t strides[3] = {K, static_cast<cuuint64_t>(kBlockK), K * rows};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(kBlockK), box_rows, kps, 1};
  cuuint32_t estride[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 output map for the small-M kernel's tile stores: dims {N, M}, box {128, box_rows}, no swizzle
// (its staging tile is row-major [token][128 columns]); rows past M and columns past N are clipped.
bool encode_bf16_tile_store_map(CUtensorMap* map, void* base, uint64_t N, uint64_t M, uint32_t box_rows) {
  cuuint64_t dims[2] = {N, M};
  cuuint64_t strides[1] = {N * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBlockM), box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_fp8_map_2d(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows) {
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBlockK), box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estride,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One instantiation per kernel, so the once-per-device flag below is per kernel.
// threads: block size.  required_regs > 0: the kernel re-splits its registers between warpgroups
// (setmaxnreg) assuming exactly that many registers per thread at launch; refuse to launch a
// build where the compiler chose another count (the split would never be granted).
// args: pointers to the kernel's arguments, in order.
template <auto KERNEL>
fg_status launch(dim3 grid, size_t smem, cudaStream_t stream, void** args, int threads, int required_regs = 0,
                 int cluster = 1) {
  // the opt-in shared-memory size is a per-function attribute: set once per device (so that a
  // call made during stream capture issues no attribute change)
  const auto kernel = KERNEL;
  static std::atomic<uint64_t> configured{0};
  const int dev = current_device();
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load(std::memory_order_acquire) & bit)) {
    if (required_regs > 0) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return FG_ERR_CUDA;
      if (fa.numRegs != required_regs) return FG_ERR_UNSUPPORTED;
    }
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess)
      return FG_ERR_CUDA;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  // programmatic dependent launch: the kernel's prologue (barriers, TMEM allocation, descriptor
  // prefetch) may overlap the previous kernel of the stream; the kernel waits for that kernel
  // (griddepcontrol.wait) before its first global-memory access
  // cluster > 1: thread-block clusters of that many CTAs along x (grid.x is a multiple of it)
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  cudaError_t e = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(kernel), args);
  if (e != cudaSuccess) return FG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FG_OK;
}

// common argument checks for the FP8 operands
fg_status check_common(const void* A, const float* sfa, const void* B, const float* sfb, const void* C, int N,
                       int K) {
  if (!A || !sfa || !B || !sfb || !C) return FG_ERR_INVALID_ARG;
  if (N < 0 || K <= 0) return FG_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % 8 != 0) return FG_ERR_ALIGNMENT;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(sfa, 16) || !aligned(sfb, 4))
    return FG_ERR_ALIGNMENT;
  return FG_OK;
}

// ------------------------------------------------------------------ runtime specialisation
// fg_set_jit(1): the tiled kernel is compiled per shape with NVRTC (fp8gemm_jit.h) and cached.
std::atomic<int> g_jit{0};
std::mutex g_jit_mutex;
// key: device, layout, tile width, stages, K blocks, K, N, sfb blocks, tile columns, grouping
typedef std::tuple<int, int, int, int, int, int, int, int, int, int> JitKey;
std::map<JitKey, CUfunction> g_jit_cache;

// The -D constants and the name expression of one specialisation of the tiled kernel.
std::vector<std::string> jit_defines(const fg::TiledParams& p) {
  std::vector<std::string> d = {"FG_JIT_NUM_KB=" + std::to_string(p.num_kb), "FG_JIT_K=" + std::to_string(p.K),
                                "FG_JIT_N=" + std::to_string(p.N), "FG_JIT_NUM_NB=" + std::to_string(p.num_nb),
                                "FG_JIT_N_BLOCKS=" + std::to_string(p.n_blocks),
                                "FG_JIT_GROUP_M=" + std::to_string(p.group_m),
                                "FG_PIPE_256=" + std::to_string(FG_PIPE_256)};
#ifdef FG_DEBUG
  d.push_back("FG_DEBUG=1");
#endif
  return d;
}
std::string jit_name(int bn, int stages, int mode) {
  const int pipe = bn > 192 ? FG_PIPE_256 : 0;
  return "fg::fp8_gemm_tiled_kernel<" + std::to_string(bn) + ", " + std::to_string(stages) + ", " +
         std::to_string(mode) + ", " + std::to_string(pipe) + ">";
}

// The specialised kernel for this call (compiled and loaded on first use), or nullptr with the
// reason in *err: FG_ERR_UNSUPPORTED without NVRTC / CUDA headers, FG_ERR_CUDA if compiling,
// loading or the register check failed.
CUfunction jit_tiled_function(int mode, int bn, int stages, size_t smem, const fg::TiledParams& p, fg_status* err) {
  std::lock_guard<std::mutex> lock(g_jit_mutex);
  const JitKey key{current_device(), mode, bn, stages, p.num_kb, p.K, p.N, p.num_nb, p.n_blocks, p.group_m};
  auto it = g_jit_cache.find(key);
  if (it != g_jit_cache.end()) return it->second;
  if (!fgjit::load_api() || !fgjit::load_driver()) {
    *err = FG_ERR_UNSUPPORTED;
    return nullptr;
  }
  std::vector<char> cubin;
  std::string lowered, log;
  const std::string name = jit_name(bn, stages, mode);
  if (!fgjit::compile("#include \"fp8_gemm_kernels.cuh\"\n", kJitHeaderCount, kJitHeaderSources, kJitHeaderNames,
                      name, jit_defines(p), &cubin, &lowered, &log)) {
    *err = FG_ERR_CUDA;
    return nullptr;
  }
  fgjit::Api& a = fgjit::api();
  CUmodule mod;
  CUfunction fn;
  int regs = 0;
  if (a.module_load(&mod, cubin.data()) != CUDA_SUCCESS || a.get_function(&fn, mod, lowered.c_str()) != CUDA_SUCCESS ||
      a.get_attr(&regs, CU_FUNC_ATTRIBUTE_NUM_REGS, fn) != CUDA_SUCCESS || regs != fg::kTiledLaunchRegs ||
      a.set_attr(fn, CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES, static_cast<int>(smem)) != CUDA_SUCCESS) {
    *err = FG_ERR_CUDA;
    return nullptr;
  }
  g_jit_cache[key] = fn;
  return fn;
}

// Launch a runtime-specialised kernel exactly as launch<>() launches the ahead-of-time one.
fg_status jit_launch(CUfunction fn, dim3 grid, int threads, size_t smem, cudaStream_t stream, void** args) {
  CUlaunchAttribute attr[1];
  attr[0].id = CU_LAUNCH_ATTRIBUTE_PROGRAMMATIC_STREAM_SERIALIZATION;
  attr[0].value.programmaticStreamSerializationAllowed = 1;
  CUlaunchConfig cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDimX = grid.x;
  cfg.gridDimY = grid.y;
  cfg.gridDimZ = grid.z;
  cfg.blockDimX = static_cast<unsigned>(threads);
  cfg.blockDimY = 1;
  cfg.blockDimZ = 1;
  cfg.sharedMemBytes = static_cast<unsigned>(smem);
  cfg.hStream = reinterpret_cast<CUstream>(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (fgjit::api().launch(&cfg, fn, args, nullptr) != CUDA_SUCCESS) return FG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FG_OK;
}

template <int MODE, int BN>
fg_status run_tiled(const Ctx* st, const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                    const int* m_indices, const int* masked_m, int M, int G, int N, int K, cudaStream_t stream,
                    int fmt_a, int fmt_b) {
  constexpr int STAGES = tiled_stages<BN>();
  fg::TiledParams p;
  p.fmt_bits = fg::idesc_formats(static_cast<uint32_t>(fmt_a), static_cast<uint32_t>(fmt_b));
  p.sfa = sfa;
  p.sfb = sfb;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.m_indices = m_indices;
  p.masked_m = masked_m;
  p.status = st->status;
  p.M = M;
  p.N = N;
  p.K = K;
  p.G = G;
  p.ld = fg_sfa_ld(M);
  p.num_kb = (K + kBlockK - 1) / kBlockK;
  p.num_nb = (N + kBlockK - 1) / kBlockK;
  p.m_blocks = (M + kBlockM - 1) / kBlockM;
  p.n_blocks = (N + BN - 1) / BN;
  p.group_m = tile_group_m(kBlockM, N, K, static_cast<long long>(p.m_blocks) * (MODE == fg::kMasked ? G : 1),
                           &p.b_resident);

  CUtensorMap mA, mB, mC;
  const uint64_t groupsA = (MODE == fg::kMasked) ? static_cast<uint64_t>(G) : 1;
  const uint64_t groupsB = (MODE == fg::kDense) ? 1 : static_cast<uint64_t>(G);
  if (!encode_fp8_map(&mA, A, K, M, groupsA, kBlockM)) return FG_ERR_CUDA;
  if (!encode_fp8_map(&mB, B, K, N, groupsB, BN)) return FG_ERR_CUDA;
  if (!encode_bf16_store_map(&mC, C, N, M, groupsA, MODE == fg::kMasked)) return FG_ERR_CUDA;

  p.ws = st->ws;
  p.counters = st->counters;
  p.counter_cap = kCounterCapacity;
  p.sk_overhead = g_tiled_sk.load(std::memory_order_relaxed);
  // masked: an upper bound (the live tiles are counted on the device)
  const long long tiles = static_cast<long long>(p.m_blocks) * p.n_blocks * (MODE == fg::kMasked ? G : 1);
  int grid = static_cast<int>(tiles < st->sms ? tiles : st->sms);
  if (tiles < st->sms && p.sk_overhead >= 0) {
    // fewer tiles than SMs: the kernel splits them in K over more CTAs if that pays (the same
    // test the kernel makes)
    const long long units = tiles * p.num_kb;
    const long long ctas = units < st->sms ? units : st->sms;
    if (fg::tiled_tail_pays(static_cast<int>(units), static_cast<int>(ctas), p.num_kb, p.sk_overhead))
      grid = static_cast<int>(ctas);
  }
  void* args[4] = {&mA, &mB, &mC, &p};
  if (g_jit.load(std::memory_order_relaxed)) {
    fg_status err = FG_OK;
    CUfunction fn = jit_tiled_function(MODE, BN, STAGES, tiled_smem_bytes<BN, STAGES>(), p, &err);
    if (!fn) return err;
    return jit_launch(fn, dim3(grid), fg::kTiledThreads, tiled_smem_bytes<BN, STAGES>(), stream, args);
  }
  return launch<fg::fp8_gemm_tiled_kernel<BN, STAGES, MODE>>(dim3(grid), tiled_smem_bytes<BN, STAGES>(), stream, args,
                                                              fg::kTiledThreads, fg::kTiledLaunchRegs);
}

// Largest number of CTA pairs of the pair kernel that can be resident at once (queried once per
// device and kernel; clusters must fit inside a GPC, so this can be below #SMs / 2).
template <auto KERNEL>
int pair_capacity(int sms, size_t smem, int threads) {
  static std::atomic<int> cached[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return sms / 2;
  int v = cached[dev].load(std::memory_order_acquire);
  if (v > 0) return v;
  // the query needs the kernel's opt-in shared-memory size in place
  if (cudaFuncSetAttribute(KERNEL, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess) {
    cudaGetLastError();
    return sms / 2;
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = smem;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, KERNEL, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sms / 2;
  }
  cached[dev].store(n, std::memory_order_release);
  return n;
}

template <int MODE, int BN, int KPS = 1, int PW = 2>
fg_status run_pair(const Ctx* st, const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                   const int* masked_m, int M, int G, int N, int K, cudaStream_t stream, int fmt_a, int fmt_b) {
  constexpr int STAGES = pair_stages<BN, KPS>();
  constexpr auto KERNEL =
      fg::fp8_gemm_pair_kernel<BN, STAGES, MODE, (BN > 192 ? FG_PIPE_256 : 0), KPS, PW>;
  using Shape = fg::PairShape<PW>;
  constexpr size_t SMEM = pair_smem_bytes<BN, STAGES, KPS>();
  fg::TiledParams p;
  p.fmt_bits = fg::idesc_formats(static_cast<uint32_t>(fmt_a), static_cast<uint32_t>(fmt_b));
  p.ws = nullptr;
  p.counters = nullptr;
  p.counter_cap = 0;
  p.sk_overhead = -1;
  p.sfa = sfa;
  p.sfb = sfb;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.m_indices = nullptr;
  p.masked_m = masked_m;
  p.status = st->status;
  p.M = M;
  p.N = N;
  p.K = K;
  p.G = G;
  p.ld = fg_sfa_ld(M);
  p.num_kb = (K + kBlockK - 1) / kBlockK;
  p.num_nb = (N + kBlockK - 1) / kBlockK;
  p.m_blocks = (M + 2 * kBlockM - 1) / (2 * kBlockM);  // 256-row blocks
  p.n_blocks = (N + BN - 1) / BN;
  p.group_m = tile_group_m(2 * kBlockM, N, K, static_cast<long long>(p.m_blocks) * (MODE == fg::kMasked ? G : 1),
                           &p.b_resident);

  CUtensorMap mA, mB, mC;
  const uint64_t groupsA = (MODE == fg::kMasked) ? static_cast<uint64_t>(G) : 1;
  const uint64_t groupsB = (MODE == fg::kDense) ? 1 : static_cast<uint64_t>(G);
  if constexpr (KPS == 1) {
    if (!encode_fp8_map(&mA, A, K, M, groupsA, kBlockM)) return FG_ERR_CUDA;
    if (!encode_fp8_map(&mB, B, K, N, groupsB, BN / 2)) return FG_ERR_CUDA;
  } else {
    if (!encode_fp8_map_kblocks_grouped(&mA, A, K, M, groupsA, kBlockM, KPS)) return FG_ERR_CUDA;
    if (!encode_fp8_map_kblocks_grouped(&mB, B, K, N, groupsB, BN / 2, KPS)) return FG_ERR_CUDA;
  }
  if (!encode_bf16_store_map(&mC, C, N, M, groupsA, MODE == fg::kMasked)) return FG_ERR_CUDA;

  const long long tiles = static_cast<long long>(p.m_blocks) * p.n_blocks * (MODE == fg::kMasked ? G : 1);
  const int cap = pair_capacity<KERNEL>(st->sms, SMEM, Shape::threads);
  const int pairs = static_cast<int>(tiles < cap ? tiles : cap);
  void* args[4] = {&mA, &mB, &mC, &p};
  return launch<KERNEL>(dim3(static_cast<unsigned>(2 * pairs)), SMEM, stream, args, Shape::threads,
                        Shape::launch_regs);
}

// Kernel and output tile width of a call of the tiled family (dense M > 128, contiguous, masked).
// The tile table (measured on B200, prefill / contiguous / masked benchmark shapes): 256-wide tiles
// run 8-13% faster than 192-wide ones (one TMEM round trip per K block stays within the register
// budget with pipelined TMEM reads, and each K block's copies carry more bytes); the CTA pair
// (256 x 256 per two SMs, each SM loading half of the weight tile) is best for dense calls unless
// its last wave is nearly empty -- it has no stream-K tail, the one-CTA kernel does -- and cannot
// serve the contiguous layout (a 256-row tile may straddle two experts).  Narrow N takes narrower
// tiles.  fg_set_dense_path (1 one-CTA, 3 pair) and fg_set_tile_n override the table.
struct TilePlan {
  int kernel;  // 1: one-CTA tiled kernel, 3: CTA-pair kernel
  int bn;      // 128, 192 or 256
};

TilePlan tile_plan(int mode, int M, int N, int G, int sms) {
  const int path = g_dense_path.load(std::memory_order_relaxed);
  const int forced = g_tile_n.load(std::memory_order_relaxed);
  TilePlan t;
  if (N <= 128) t = {1, 128};
  else if (N <= 192) t = {1, 192};
  else if (mode != fg::kDense) t = {1, 256};
  else {
    const long long pair_tiles = static_cast<long long>((M + 255) / 256) * ((N + 255) / 256);
    const int pairs = sms / 2 > 0 ? sms / 2 : 1;
    const long long rem = pair_tiles % pairs;
    // a last wave holding at most a quarter of the pairs: the one-CTA kernel's stream-K tail wins
    t = (rem != 0 && rem * 4 <= pairs) ? TilePlan{1, 256} : TilePlan{3, 256};
    (void)G;
  }
  if (path == 1) t.kernel = 1;
  if (path == 3 && mode != fg::kContiguous) t.kernel = 3;
  if (forced != 0) t.bn = forced;
  if (t.kernel == 3 && t.bn != 256) t.bn = 192;  // the pair kernel has 192 and 256
  return t;
}

template <int MODE>
fg_status dispatch_tiled(const Ctx* st, const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                         const int* m_indices, const int* masked_m, int M, int G, int N, int K, cudaStream_t stream,
                         int fmt_a, int fmt_b) {
  const TilePlan t = tile_plan(MODE, M, N, G, st->sms);
  if (t.kernel == 3 && MODE != fg::kContiguous) {
    constexpr int PM = MODE == fg::kContiguous ? fg::kDense : MODE;  // (never the contiguous layout)
    const bool pairs = pair_kps_for(K) == 2;
    if (t.bn == 256 && g_pair_pw.load(std::memory_order_relaxed) == 4)
      return pairs ? run_pair<PM, 256, 2, 4>(st, A, sfa, B, sfb, C, masked_m, M, G, N, K, stream, fmt_a, fmt_b)
                   : run_pair<PM, 256, 1, 4>(st, A, sfa, B, sfb, C, masked_m, M, G, N, K, stream, fmt_a, fmt_b);
    if (t.bn == 256)
      return pairs ? run_pair<PM, 256, 2>(st, A, sfa, B, sfb, C, masked_m, M, G, N, K, stream, fmt_a, fmt_b)
                   : run_pair<PM, 256, 1>(st, A, sfa, B, sfb, C, masked_m, M, G, N, K, stream, fmt_a, fmt_b);
    return pairs ? run_pair<PM, kPairBN, 2>(st, A, sfa, B, sfb, C, masked_m, M, G, N, K, stream, fmt_a, fmt_b)
                 : run_pair<PM, kPairBN, 1>(st, A, sfa, B, sfb, C, masked_m, M, G, N, K, stream, fmt_a, fmt_b);
  }
  if (t.bn == 128)
    return run_tiled<MODE, 128>(st, A, sfa, B, sfb, C, m_indices, masked_m, M, G, N, K, stream, fmt_a, fmt_b);
  if (t.bn == 256)
    return run_tiled<MODE, 256>(st, A, sfa, B, sfb, C, m_indices, masked_m, M, G, N, K, stream, fmt_a, fmt_b);
  return run_tiled<MODE, kTiledBN>(st, A, sfa, B, sfb, C, m_indices, masked_m, M, G, N, K, stream, fmt_a, fmt_b);
}

// Largest number of clusters of `size` CTAs of KERNEL that can be resident at once (clusters must
// fit inside a GPC, so this can be below #SMs / size); queried once per device, kernel and size.
template <auto KERNEL>
int cluster_capacity(int size, int threads, size_t smem) {
  static std::atomic<int> cached[kMaxDevices][4];
  const int dev = current_device();
  const int slot = size == 2 ? 0 : size == 4 ? 1 : size == 8 ? 2 : 3;
  if (dev < 0 || dev >= kMaxDevices || slot == 3) return 0;
  int v = cached[dev][slot].load(std::memory_order_acquire);
  if (v != 0) return v < 0 ? 0 : v;
  // the query needs the kernel's opt-in shared-memory size in place
  if (cudaFuncSetAttribute(KERNEL, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(size);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(size), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, KERNEL, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 0;
  }
  cached[dev][slot].store(n > 0 ? n : -1, std::memory_order_release);
  return n;
}

struct SwapChoice {
  int grid;
  int tile_aligned;
  int cluster;
};

// Schedule of the small-M kernel for n_tiles weight tiles of 128 rows and num_kb K blocks.
// Whole tiles instead of stream-K when that costs at most kSplitOverheadUnits more K blocks on the
// busiest CTA than the even split of the units (the split-K publication and fix-up cost about
// that much on the decode shapes).  Cluster split-K: S CTAs per tile, all tiles resident at once
// (tiles <= the cluster capacity), each CTA with at least one K block.  Cost model in K blocks on
// the busiest CTA: the cluster split pays ceil(KB / S) + FG_SWAP_CLUSTER_UNITS; stream-K its share
// + FG_SWAP_STREAMK_UNITS (publishing a partial through global memory and the last CTA's sum of
// the pieces); tile-aligned ranges their whole tiles.
#ifndef FG_SPLIT_OVERHEAD_UNITS
#define FG_SPLIT_OVERHEAD_UNITS 8
#endif
#ifndef FG_SWAP_CLUSTER_UNITS
#define FG_SWAP_CLUSTER_UNITS 2
#endif
#ifndef FG_SWAP_STREAMK_UNITS
#define FG_SWAP_STREAMK_UNITS 16
#endif
// Units are groups of KPS K blocks (the last of a tile may be shorter); costs are in K blocks.
template <int MP, int KPS = 1>
SwapChoice swap_choose(int sms, int n_tiles, int num_kb_blocks) {
  constexpr int STAGES = swap_stages<MP, KPS>();
  constexpr auto KERNEL = fg::fp8_gemm_swap_streamk_kernel<MP, STAGES, KPS>;
  constexpr size_t SMEM = swap_smem_bytes<MP, STAGES, KPS>();
  constexpr long long kSplitOverheadUnits = FG_SPLIT_OVERHEAD_UNITS;
  const int num_kb = (num_kb_blocks + KPS - 1) / KPS;  // units per tile
  SwapChoice c;
  const long long units = static_cast<long long>(n_tiles) * num_kb;
  c.grid = static_cast<int>(units < sms ? units : sms);
  const long long aligned_units = (n_tiles + sms - 1) / sms * static_cast<long long>(num_kb_blocks);
  const long long split_units = (units + c.grid - 1) / c.grid * KPS;
  c.tile_aligned = (n_tiles >= sms && aligned_units <= split_units + kSplitOverheadUnits) ? 1 : 0;
  if (c.tile_aligned) c.grid = sms;
  c.cluster = 1;
  const int sched = g_swap_schedule.load(std::memory_order_relaxed);
  if (sched == 1) {  // whole tiles, one CTA per tile up to the SM count
    c.tile_aligned = 1;
    c.grid = n_tiles < sms ? n_tiles : sms;
    return c;
  }
  if (sched == 0 || sched > 1) {
    long long best = c.tile_aligned ? aligned_units : (split_units + (num_kb > 1 ? FG_SWAP_STREAMK_UNITS : 0));
    for (int S : {8, 4, 2}) {
      if (sched > 0 && S != sched) continue;
      if (S > num_kb || n_tiles > cluster_capacity<KERNEL>(S, fg::kThreads, SMEM)) continue;
      const long long cost = (num_kb + S - 1) / S * KPS + FG_SWAP_CLUSTER_UNITS;
      if (sched > 0 || cost < best) {
        best = cost;
        c.cluster = S;
      }
    }
  }
  if (c.cluster > 1) {
    c.tile_aligned = 0;
    c.grid = n_tiles * c.cluster;
  }
  return c;
}

template <int MP, int KPS>
fg_status run_swap_t(const Ctx* st, const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                     int M, int N, int K, cudaStream_t stream, int fmt_a, int fmt_b, unsigned flags) {
  constexpr int STAGES = swap_stages<MP, KPS>();
  fg::SwapParams p;
  // swap-AB: the MMA's A operand is the weight tile (B of the GEMM), its B operand the tokens
  p.fmt_bits = fg::idesc_formats(static_cast<uint32_t>(fmt_b), static_cast<uint32_t>(fmt_a));
  p.sfa = sfa;
  p.sfb = sfb;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.ws = st->ws;
  p.counters = st->counters;
  p.counter_cap = kCounterCapacity;
  p.status = st->status;
  p.M = M;
  p.N = N;
  p.K = K;
  p.ld = fg_sfa_ld(M);
  p.num_kb = (K + kBlockK - 1) / kBlockK;
  p.n_tiles = (N + kBlockM - 1) / kBlockM;
  p.debug_stall = g_debug_stall.load(std::memory_order_relaxed);
  p.static_b = (flags & FG_FLAG_STATIC_B) ? 1 : 0;
  if (p.n_tiles > kCounterCapacity) return FG_ERR_UNSUPPORTED;

  CUtensorMap mW, mT, mC;
  if constexpr (KPS == 1) {
    if (!encode_fp8_map_2d(&mW, B, K, N, kBlockM)) return FG_ERR_CUDA;
    if (!encode_fp8_map_2d(&mT, A, K, M, MP)) return FG_ERR_CUDA;
  } else {
    if (!encode_fp8_map_kblocks(&mW, B, K, N, kBlockM, KPS)) return FG_ERR_CUDA;
    if (!encode_fp8_map_kblocks(&mT, A, K, M, MP, KPS)) return FG_ERR_CUDA;
  }
  if (!encode_bf16_tile_store_map(&mC, C, N, M, MP)) return FG_ERR_CUDA;
  const SwapChoice c = swap_choose<MP, KPS>(st->sms, p.n_tiles, p.num_kb);
  p.tile_aligned = c.tile_aligned;
  p.cluster = c.cluster;
  void* args[4] = {&mW, &mT, &mC, &p};
  return launch<fg::fp8_gemm_swap_streamk_kernel<MP, STAGES, KPS>>(
      dim3(c.grid), swap_smem_bytes<MP, STAGES, KPS>(), stream, args, fg::kThreads, 0, c.cluster);
}

// K blocks per stage for a small-M call: 2 when K is a multiple of 128 (the 3-D copies need whole
// K blocks) and has at least 4 of them (so that a tile still splits into two or more units for the
// cluster and stream-K schedules), unless fg_set_stage_kblocks says otherwise (2: whenever K allows).
int swap_kps_for(int K) {
  const int f = g_stage_kb.load(std::memory_order_relaxed);
  if (K % kBlockK != 0 || f == 1) return 1;
  return (f == 2 || K / kBlockK >= 4) ? 2 : 1;
}

template <int MP>
fg_status run_swap(const Ctx* st, const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                   int M, int N, int K, cudaStream_t stream, int fmt_a, int fmt_b, unsigned flags) {
  if (swap_kps_for(K) == 2)
    return run_swap_t<MP, 2>(st, A, sfa, B, sfb, C, M, N, K, stream, fmt_a, fmt_b, flags);
  return run_swap_t<MP, 1>(st, A, sfa, B, sfb, C, M, N, K, stream, fmt_a, fmt_b, flags);
}

// ---------------------------------------------------------------------------------------------
// Allocation-free variant of the dense small-M (swap-AB stream-K) path.  Its split-K scratch
// (partial tiles, per-tile arrival counters and a status word) lives in this file-scope device
// array, so the entry point never allocates.  Every GPU that loads the library holds the array
// until the process exits.  In host code `g_noalloc_scratch` is only a host-side stand-in for
// the symbol: the device address is obtained with cudaGetSymbolAddress, once per device.
constexpr size_t kNoAllocPartialBytes = size_t(16) << 20;  // split-K partial tiles
constexpr int kNoAllocCounters = 1 << 14;                  // n-tiles: N <= 2,097,152
constexpr size_t kNoAllocBytes = kNoAllocPartialBytes + kNoAllocCounters * sizeof(int) + 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

struct NoAllocDevice {
  std::atomic<bool> ready{false};  // published (release) after sms and base are set
  int sms = 0;
  unsigned char* base = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocDevice g_noalloc[kMaxDevices];

fg_status noalloc_setup(int dev, NoAllocDevice** out) {
  NoAllocDevice& d = g_noalloc[dev];
  if (!d.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!d.ready.load(std::memory_order_relaxed)) {
      if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
          return FG_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
      int major = 0, minor = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return FG_ERR_CUDA;
      if (major != 10 || minor != 0) return FG_ERR_UNSUPPORTED;  // built for sm_100a only, as fg_init
      if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FG_ERR_CUDA;
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return FG_ERR_CUDA;
      d.base = static_cast<unsigned char*>(ptr);
      d.ready.store(true, std::memory_order_release);
    }
  }
  *out = &d;
  return FG_OK;
}

template <int MP>
fg_status run_swap_noalloc(const NoAllocDevice& d, const void* A, const float* sfa, const void* B, const float* sfb,
                           void* C, int M, int N, int K, cudaStream_t stream) {
  constexpr int STAGES = swap_stages<MP>();
  fg::SwapParams p;
  p.sfa = sfa;
  p.sfb = sfb;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.ws = reinterpret_cast<float*>(d.base);
  p.counters = reinterpret_cast<int*>(d.base + kNoAllocPartialBytes);
  p.counter_cap = kNoAllocCounters;
  p.status = p.counters + kNoAllocCounters;
  p.M = M;
  p.N = N;
  p.K = K;
  p.ld = fg_sfa_ld(M);
  p.num_kb = (K + kBlockK - 1) / kBlockK;
  p.n_tiles = (N + kBlockM - 1) / kBlockM;
  p.debug_stall = g_debug_stall.load(std::memory_order_relaxed);
  p.fmt_bits = 0;  // e4m3 x e4m3
  p.tile_aligned = 0;
  p.cluster = 1;
  p.static_b = 0;
  if (p.n_tiles > kNoAllocCounters) return FG_ERR_UNSUPPORTED;
  // the counters must start at zero; the kernel leaves them at zero, but a call that gave up a
  // wait may not have, so clear the ones this call uses (a memset, no allocation)
  if (cudaMemsetAsync(p.counters, 0, static_cast<size_t>(p.n_tiles) * sizeof(int), stream) != cudaSuccess)
    return FG_ERR_CUDA;
  CUtensorMap mW, mT, mC;
  if (!encode_fp8_map_2d(&mW, B, K, N, kBlockM)) return FG_ERR_CUDA;
  if (!encode_fp8_map_2d(&mT, A, K, M, MP)) return FG_ERR_CUDA;
  if (!encode_bf16_tile_store_map(&mC, C, N, M, MP)) return FG_ERR_CUDA;
  // the partial tiles (two per CTA) must fit in the array: that caps the grid, not the problem size
  const long long cap = static_cast<long long>(kNoAllocPartialBytes / (2 * MP * kBlockM * sizeof(float)));
  long long grid = static_cast<long long>(p.n_tiles) * p.num_kb;
  if (grid > d.sms) grid = d.sms;
  if (grid > cap) grid = cap;
  void* args[4] = {&mW, &mT, &mC, &p};
  return launch<fg::fp8_gemm_swap_streamk_kernel<MP, STAGES>>(dim3(static_cast<unsigned>(grid)),
                                                               swap_smem_bytes<MP, STAGES>(), stream, args,
                                                               fg::kThreads);
}

}  // namespace

extern "C" {

fg_status fg_init(int device) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (device < 0 || device >= kMaxDevices) return FG_ERR_INVALID_ARG;
  if (cudaSetDevice(device) != cudaSuccess) return FG_ERR_CUDA;
  DeviceState& st = g_dev[device];
  if (st.ready) return FG_OK;
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return FG_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess)
    return FG_ERR_CUDA;
  if (major != 10 || minor != 0) return FG_ERR_UNSUPPORTED;  // built for sm_100a only
  if (cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return FG_ERR_CUDA;
  // two partial tiles per CTA: MP x 128 (swap kernel) or 128 x BN (tiled kernel's stream-K tail)
  if (cudaMalloc(&st.status, sizeof(int)) != cudaSuccess) return FG_ERR_CUDA;
  if (cudaMalloc(&st.ws, workspace_partial_bytes(st.sms)) != cudaSuccess) return FG_ERR_CUDA;
  if (cudaMalloc(&st.counters, kCounterCapacity * sizeof(int)) != cudaSuccess) return FG_ERR_CUDA;
  if (cudaMemset(st.status, 0, sizeof(int)) != cudaSuccess) return FG_ERR_CUDA;
  if (cudaMemset(st.counters, 0, kCounterCapacity * sizeof(int)) != cudaSuccess) return FG_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return FG_ERR_CUDA;
  st.ready = true;
  return FG_OK;
}

void fg_shutdown(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  int prev = -1;
  cudaGetDevice(&prev);
  for (int d = 0; d < kMaxDevices; ++d) {
    DeviceState& st = g_dev[d];
    if (!st.ready) continue;
    cudaSetDevice(d);
    cudaFree(st.status);
    cudaFree(st.ws);
    cudaFree(st.counters);
    st = DeviceState();
  }
  if (prev >= 0) cudaSetDevice(prev);
}

int fg_m_alignment(void) { return kBlockM; }

int fg_sfa_ld(int M) { return M <= 0 ? 0 : (M + 3) / 4 * 4; }

int fg_set_dense_path(int path) {
  if (path < 0 || path > 3) return g_dense_path.load();
  return g_dense_path.exchange(path);
}

uint64_t fg_launch_count(void) { return g_launches.load(); }

int fg_debug_set_stall(int enable) { return g_debug_stall.exchange(enable ? 1 : 0); }

int fg_tile_plan(int layout, int M, int N, int K, int G) {
  if (layout < 0 || layout > 2 || M <= 0 || N <= 0 || K <= 0 || G <= 0) return -1;
  fg_status err;
  const DeviceState* st = state_for_current(&err);
  if (!st) return -1;
  const int path = g_dense_path.load();
  if (layout == 0 && (path == 2 || (path == 0 && M <= kMaxSwapMP))) return 2000;
  const TilePlan t = tile_plan(layout, M, N, G, st->sms);
  return t.kernel * 1000 + t.bn;
}

int fg_set_tile_order(int order) {
  if (order < 0 || order > 2) return g_tile_order.load();
  return g_tile_order.exchange(order);
}

int fg_set_tile_n(int bn) {
  if (bn != 0 && bn != 128 && bn != 192 && bn != 256) return g_tile_n.load();
  return g_tile_n.exchange(bn);
}

int fg_set_tiled_streamk(int overhead) { return g_tiled_sk.exchange(overhead < 0 ? -1 : overhead); }

int fg_swap_plan(int M, int N, int K) {
  if (M <= 0 || M > kMaxSwapMP || N <= 0 || K <= 0) return -1;
  fg_status err;
  DeviceState* st = state_for_current(&err);
  if (!st) return -1;
  const int tiles = (N + kBlockM - 1) / kBlockM;
  const int kb = (K + kBlockK - 1) / kBlockK;
  SwapChoice c;
  if (swap_kps_for(K) == 2)
    c = M <= 32 ? swap_choose<32, 2>(st->sms, tiles, kb)
                : M <= 64 ? swap_choose<64, 2>(st->sms, tiles, kb) : swap_choose<128, 2>(st->sms, tiles, kb);
  else
    c = M <= 32 ? swap_choose<32, 1>(st->sms, tiles, kb)
                : M <= 64 ? swap_choose<64, 1>(st->sms, tiles, kb) : swap_choose<128, 1>(st->sms, tiles, kb);
  return c.cluster > 1 ? c.cluster : c.tile_aligned;
}

int fg_set_jit(int enable) { return g_jit.exchange(enable ? 1 : 0); }

int fg_jit_cache_size(void) {
  std::lock_guard<std::mutex> lock(g_jit_mutex);
  return static_cast<int>(g_jit_cache.size());
}

fg_status fg_jit_compile_check(int bn, int num_kb, int N, size_t* cubin_bytes) {
  if (!cubin_bytes || num_kb <= 0 || N <= 0 || (bn != 128 && bn != 192 && bn != 256)) return FG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_jit_mutex);
  if (!fgjit::load_api()) return FG_ERR_UNSUPPORTED;
  fg::TiledParams p;
  std::memset(&p, 0, sizeof(p));
  p.num_kb = num_kb;
  p.K = num_kb * kBlockK;
  p.N = N;
  p.num_nb = (N + kBlockK - 1) / kBlockK;
  p.n_blocks = (N + bn - 1) / bn;
  p.group_m = 1;
  const int stages = bn == 128 ? tiled_stages<128>() : (bn == 192 ? tiled_stages<192>() : tiled_stages<256>());
  std::vector<char> cubin;
  std::string lowered, log;
  if (!fgjit::compile("#include \"fp8_gemm_kernels.cuh\"\n", kJitHeaderCount, kJitHeaderSources, kJitHeaderNames,
                      jit_name(bn, stages, fg::kDense), jit_defines(p), &cubin, &lowered, &log))
    return FG_ERR_CUDA;
  *cubin_bytes = cubin.size();
  return FG_OK;
}

int fg_set_pair_promotion(int warpgroups) {
  if (warpgroups != 2 && warpgroups != 4) return g_pair_pw.load();
  return g_pair_pw.exchange(warpgroups);
}

int fg_set_stage_kblocks(int kps) {
  if (kps != 0 && kps != 1 && kps != 2) return g_stage_kb.load();
  return g_stage_kb.exchange(kps);
}

int fg_set_swap_schedule(int schedule) {
  if (schedule != 0 && schedule != -1 && schedule != 1 && schedule != 2 && schedule != 4 && schedule != 8)
    return g_swap_schedule.load();
  return g_swap_schedule.exchange(schedule);
}

static bool valid_formats(int fmt_a, int fmt_b) {
  return (fmt_a == FG_E4M3 || fmt_a == FG_E5M2) && (fmt_b == FG_E4M3 || fmt_b == FG_E5M2);
}

size_t fg_workspace_bytes(void) {
  fg_status s;
  const DeviceState* st = state_for_current(&s);
  return st ? workspace_bytes_for(st->sms) : 0;
}

// Launch context of a call: the library's workspace (workspace == NULL, workspace_bytes == 0) or
// the caller's (at least fg_workspace_bytes(), 16-byte aligned).
static fg_status resolve_ctx(void* workspace, size_t workspace_bytes, Ctx* out) {
  fg_status s;
  const DeviceState* st = state_for_current(&s);
  if (!st) return s;
  *out = ctx_of(st);
  if (workspace == nullptr) return workspace_bytes == 0 ? FG_OK : FG_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return FG_ERR_ALIGNMENT;
  if (workspace_bytes < workspace_bytes_for(st->sms)) return FG_ERR_INVALID_ARG;
  out->ws = static_cast<float*>(workspace);
  out->counters = reinterpret_cast<int*>(static_cast<char*>(workspace) + workspace_partial_bytes(st->sms));
  return FG_OK;
}

fg_status fp8_gemm_nt_ws(const void* A, const float* sfa, const void* B, const float* sfb, void* C, int M, int N,
                         int K, int fmt_a, int fmt_b, unsigned flags, void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (M < 0 || N < 0 || !valid_formats(fmt_a, fmt_b) || (flags & ~kKnownFlags)) return FG_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FG_OK;
  fg_status s = check_common(A, sfa, B, sfb, C, N, K);
  if (s != FG_OK) return s;
  if (static_cast<long long>(M) * K >= (1ll << 40) || static_cast<long long>(N) * K >= (1ll << 40))
    return FG_ERR_UNSUPPORTED;
  Ctx ctx;
  s = resolve_ctx(workspace, workspace_bytes, &ctx);
  if (s != FG_OK) return s;
  const Ctx* st = &ctx;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int path = g_dense_path.load();
  const bool swap = (path == 2) || (path == 0 && M <= kMaxSwapMP);
  if (swap) {
    if (M > kMaxSwapMP) return FG_ERR_UNSUPPORTED;
    if (M <= 32) return run_swap<32>(st, A, sfa, B, sfb, C, M, N, K, cs, fmt_a, fmt_b, flags);
    if (M <= 64) return run_swap<64>(st, A, sfa, B, sfb, C, M, N, K, cs, fmt_a, fmt_b, flags);
    return run_swap<128>(st, A, sfa, B, sfb, C, M, N, K, cs, fmt_a, fmt_b, flags);
  }
  return dispatch_tiled<fg::kDense>(st, A, sfa, B, sfb, C, nullptr, nullptr, M, 1, N, K, cs, fmt_a, fmt_b);
}

fg_status fp8_gemm_nt_ex(const void* A, const float* sfa, const void* B, const float* sfb, void* C, int M, int N,
                         int K, int fmt_a, int fmt_b, void* stream) {
  return fp8_gemm_nt_ws(A, sfa, B, sfb, C, M, N, K, fmt_a, fmt_b, 0u, nullptr, 0, stream);
}

fg_status fp8_gemm_nt(const void* A, const float* sfa, const void* B, const float* sfb, void* C, int M, int N,
                      int K, void* stream) {
  return fp8_gemm_nt_ex(A, sfa, B, sfb, C, M, N, K, FG_E4M3, FG_E4M3, stream);
}

fg_status fp8_gemm_grouped_contiguous_ws(const void* A, const float* sfa, const void* B, const float* sfb,
                                         void* C, const int* m_indices, int M_total, int G, int N, int K, int fmt_a,
                                         int fmt_b, unsigned flags, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  if (M_total < 0 || N < 0 || G < 0 || !valid_formats(fmt_a, fmt_b) || (flags & ~kKnownFlags))
    return FG_ERR_INVALID_ARG;
  if (M_total == 0 || N == 0) return FG_OK;
  if (G == 0) return FG_ERR_INVALID_ARG;
  fg_status s = check_common(A, sfa, B, sfb, C, N, K);
  if (s != FG_OK) return s;
  if (!m_indices) return FG_ERR_INVALID_ARG;
  if (!aligned(m_indices, 4)) return FG_ERR_ALIGNMENT;
  if (static_cast<long long>(M_total) * K >= (1ll << 40) || static_cast<long long>(G) * N * K >= (1ll << 40))
    return FG_ERR_UNSUPPORTED;
  Ctx ctx;
  s = resolve_ctx(workspace, workspace_bytes, &ctx);
  if (s != FG_OK) return s;
  return dispatch_tiled<fg::kContiguous>(&ctx, A, sfa, B, sfb, C, m_indices, nullptr, M_total, G, N, K,
                                    static_cast<cudaStream_t>(stream), fmt_a, fmt_b);
}

fg_status fp8_gemm_grouped_contiguous_ex(const void* A, const float* sfa, const void* B, const float* sfb,
                                         void* C, const int* m_indices, int M_total, int G, int N, int K, int fmt_a,
                                         int fmt_b, void* stream) {
  return fp8_gemm_grouped_contiguous_ws(A, sfa, B, sfb, C, m_indices, M_total, G, N, K, fmt_a, fmt_b, 0u, nullptr,
                                        0, stream);
}

fg_status fp8_gemm_grouped_contiguous(const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                                      const int* m_indices, int M_total, int G, int N, int K, void* stream) {
  return fp8_gemm_grouped_contiguous_ex(A, sfa, B, sfb, C, m_indices, M_total, G, N, K, FG_E4M3, FG_E4M3, stream);
}

fg_status fp8_gemm_grouped_masked_ws(const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                                     const int* masked_m, int G, int Mmax, int N, int K, int fmt_a, int fmt_b,
                                     unsigned flags, void* workspace, size_t workspace_bytes, void* stream) {
  if (G < 0 || Mmax < 0 || N < 0 || !valid_formats(fmt_a, fmt_b) || (flags & ~kKnownFlags))
    return FG_ERR_INVALID_ARG;
  if (G == 0 || Mmax == 0 || N == 0) return FG_OK;
  fg_status s = check_common(A, sfa, B, sfb, C, N, K);
  if (s != FG_OK) return s;
  if (!masked_m) return FG_ERR_INVALID_ARG;
  if (!aligned(masked_m, 4)) return FG_ERR_ALIGNMENT;
  if (G > fg::kMaskedMaxGroups) return FG_ERR_UNSUPPORTED;
  if (static_cast<long long>(G) * Mmax * K >= (1ll << 40) || static_cast<long long>(G) * N * K >= (1ll << 40))
    return FG_ERR_UNSUPPORTED;
  Ctx ctx;
  s = resolve_ctx(workspace, workspace_bytes, &ctx);
  if (s != FG_OK) return s;
  return dispatch_tiled<fg::kMasked>(&ctx, A, sfa, B, sfb, C, nullptr, masked_m, Mmax, G, N, K,
                                static_cast<cudaStream_t>(stream), fmt_a, fmt_b);
}

fg_status fp8_gemm_grouped_masked_ex(const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                                     const int* masked_m, int G, int Mmax, int N, int K, int fmt_a, int fmt_b,
                                     void* stream) {
  return fp8_gemm_grouped_masked_ws(A, sfa, B, sfb, C, masked_m, G, Mmax, N, K, fmt_a, fmt_b, 0u, nullptr, 0,
                                     stream);
}

fg_status fp8_gemm_grouped_masked(const void* A, const float* sfa, const void* B, const float* sfb, void* C,
                                  const int* masked_m, int G, int Mmax, int N, int K, void* stream) {
  return fp8_gemm_grouped_masked_ex(A, sfa, B, sfb, C, masked_m, G, Mmax, N, K, FG_E4M3, FG_E4M3, stream);
}

fg_status fp8_gemm_nt_noalloc(const void* A, const float* sfa, const void* B, const float* sfb, void* C, int M,
                              int N, int K, void* stream) {
  if (M < 0 || N < 0) return FG_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FG_OK;
  fg_status s = check_common(A, sfa, B, sfb, C, N, K);
  if (s != FG_OK) return s;
  if (M > kMaxSwapMP) return FG_ERR_UNSUPPORTED;  // only the small-M kernel has this variant
  if (static_cast<long long>(M) * K >= (1ll << 40) || static_cast<long long>(N) * K >= (1ll << 40))
    return FG_ERR_UNSUPPORTED;
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return FG_ERR_CUDA;
  NoAllocDevice* d = nullptr;
  s = noalloc_setup(dev, &d);
  if (s != FG_OK) return s;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (M <= 32) return run_swap_noalloc<32>(*d, A, sfa, B, sfb, C, M, N, K, cs);
  if (M <= 64) return run_swap_noalloc<64>(*d, A, sfa, B, sfb, C, M, N, K, cs);
  return run_swap_noalloc<128>(*d, A, sfa, B, sfb, C, M, N, K, cs);
}

fg_status fg_noalloc_status(void* stream) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices || !g_noalloc[dev].ready.load(std::memory_order_acquire))
    return FG_OK;  // never called here
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FG_ERR_CUDA;
  int* status = reinterpret_cast<int*>(g_noalloc[dev].base + kNoAllocPartialBytes) + kNoAllocCounters;
  int v = 0;
  if (cudaMemcpy(&v, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FG_ERR_CUDA;
  if (v != 0 && cudaMemset(status, 0, sizeof(int)) != cudaSuccess) return FG_ERR_CUDA;
  return static_cast<fg_status>(v);
}

// ---------------------------------------------------------------------------- the cast step
namespace {
int sm_count_of_current() {
  static std::atomic<int> cached[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int v = cached[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return 0;
  cached[dev].store(v, std::memory_order_relaxed);
  return v;
}
}  // namespace

fg_status fp8_cast_rows_ex(const void* X, void* Q, float* sfa, int G, int M, int K, int fmt, void* stream) {
  if (!X || !Q || !sfa || G < 0 || M < 0 || K < 0 || (fmt != FG_E4M3 && fmt != FG_E5M2)) return FG_ERR_INVALID_ARG;
  if (G == 0 || M == 0 || K == 0) return FG_OK;
  if (K % 16 != 0 || !aligned(X, 16) || !aligned(Q, 16) || !aligned(sfa, 4)) return FG_ERR_ALIGNMENT;
  if (static_cast<long long>(G) * M * K >= (1ll << 40)) return FG_ERR_UNSUPPORTED;
  const int sms = sm_count_of_current();
  if (sms <= 0) return FG_ERR_CUDA;
  const long long rows = static_cast<long long>(G) * M;
  const int chunks = (K + 256 * fg::kCastSpans - 1) / (256 * fg::kCastSpans);
  const long long warps = rows * chunks;
  long long blocks = (warps + 7) / 8;
  if (blocks > 8ll * sms) blocks = 8ll * sms;
  // a plain (fully stream-ordered) launch: the kernel does not wait for a preceding grid itself
  const auto kernel = fmt == FG_E4M3 ? fg::fp8_cast_rows_kernel<0> : fg::fp8_cast_rows_kernel<1>;
  kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(X), static_cast<uint8_t*>(Q), sfa, M, K, fg_sfa_ld(M), rows, chunks);
  if (cudaGetLastError() != cudaSuccess) return FG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FG_OK;
}

fg_status fp8_cast_rows(const void* X, void* Q, float* sfa, int G, int M, int K, void* stream) {
  return fp8_cast_rows_ex(X, Q, sfa, G, M, K, FG_E4M3, stream);
}

fg_status fp8_cast_blocks_ex(const void* X, void* Q, float* sfb, int G, int N, int K, int fmt, void* stream) {
  if (!X || !Q || !sfb || G < 0 || N < 0 || K < 0 || (fmt != FG_E4M3 && fmt != FG_E5M2)) return FG_ERR_INVALID_ARG;
  if (G == 0 || N == 0 || K == 0) return FG_OK;
  if (K % 16 != 0 || !aligned(X, 16) || !aligned(Q, 16) || !aligned(sfb, 4)) return FG_ERR_ALIGNMENT;
  if (static_cast<long long>(G) * N * K >= (1ll << 40) || G > 65535 || (N + 127) / 128 > 65535)
    return FG_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>((K + 127) / 128), static_cast<unsigned>((N + 127) / 128),
                  static_cast<unsigned>(G));
  const auto kernel = fmt == FG_E4M3 ? fg::fp8_cast_blocks_kernel<0> : fg::fp8_cast_blocks_kernel<1>;
  kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const __nv_bfloat16*>(X),
                                                              static_cast<uint8_t*>(Q), sfb, N, K);
  if (cudaGetLastError() != cudaSuccess) return FG_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FG_OK;
}

fg_status fp8_cast_blocks(const void* X, void* Q, float* sfb, int G, int N, int K, void* stream) {
  return fp8_cast_blocks_ex(X, Q, sfb, G, N, K, FG_E4M3, stream);
}

fg_status fg_get_device_status(void* stream) {
  fg_status s;
  DeviceState* st = state_for_current(&s);
  if (!st) return s;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, st->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FG_ERR_CUDA;
  if (v != 0) {
    // a kernel gave up early: clear the word and the stream-K counters it may have left behind
    if (cudaMemset(st->status, 0, sizeof(int)) != cudaSuccess) return FG_ERR_CUDA;
    if (cudaMemset(st->counters, 0, kCounterCapacity * sizeof(int)) != cudaSuccess) return FG_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return FG_ERR_CUDA;
    return static_cast<fg_status>(v);
  }
  return FG_OK;
}

const char* fg_status_string(fg_status status) {
  switch (status) {
    case FG_OK: return "FG_OK";
    case FG_ERR_INVALID_ARG: return "FG_ERR_INVALID_ARG";
    case FG_ERR_ALIGNMENT: return "FG_ERR_ALIGNMENT";
    case FG_ERR_UNSUPPORTED: return "FG_ERR_UNSUPPORTED";
    case FG_ERR_NOT_INITIALIZED: return "FG_ERR_NOT_INITIALIZED";
    case FG_ERR_CUDA: return "FG_ERR_CUDA";
    case FG_ERR_TIMEOUT: return "FG_ERR_TIMEOUT";
    case FG_ERR_DEVICE_CHECK: return "FG_ERR_DEVICE_CHECK";
  }
  return "FG_ERR_UNKNOWN";
}

}  // extern "C"
