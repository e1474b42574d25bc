// Host side of the C ABI declared in include/vrar.h: argument checks, the
// per-device workspace, grid sizing, the per-size selector and the status
// word. Every call queues exactly one kernel on the caller's stream.

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kernels.cuh"
#include "vrar.h"

namespace vrar {
namespace {

constexpr int kMaxDevices = 64;

struct Settings {
  std::atomic<int> group_size{8};
  std::atomic<int> rd_chunks{4};
  std::atomic<int> edge_sync{0};
  std::atomic<uint64_t> timeout_ns{2000000000ull};
  std::atomic<uint32_t> fault_mask{0};
  std::atomic<int> spin_stats{0};
  std::atomic<int> max_ctas{0};  // grid cap per call, 0 = none
  std::atomic<int> payload_wire{VRAR_WIRE_ELEMENT};
  std::atomic<int> fp8_quant{0};
};
Settings g_set;

// Library-owned device memory of one device: control words, the three
// signal arrays and the payload slots, zeroed when allocated.
struct Workspace {
  uint32_t* ctrl = nullptr;  // kCtrlWords words, then kPhases * kSigPhaseWords signal words
  uint32_t* sig = nullptr;
  uint64_t* ll = nullptr;
  size_t ll_bytes = 0;
  int sms = 0;
};

std::mutex g_mu;
Workspace g_ws[kMaxDevices];

bool valid_dtype(vrar_dtype_t dt) { return dt == VRAR_BF16 || dt == VRAR_FP32 || dt == VRAR_FP16; }
size_t elem_size(vrar_dtype_t dt) { return dt == VRAR_FP32 ? 4 : 2; }
int64_t per_item(vrar_dtype_t dt) { return dt == VRAR_FP32 ? 4 : 8; }
bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int ilog2(int x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return s;
}

int cuda_fail(cudaError_t e) {
  (void)e;
  cudaGetLastError();  // clear the non-sticky error so later calls start clean
  return VRAR_ECUDA;
}

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (*dev < 0 || *dev >= kMaxDevices) return VRAR_ECUDA;
  return VRAR_OK;
}

// Allocate (once) the control + signal block and grow the payload slots to at
// least ll_need bytes. Growing frees the old slots after a device-wide sync.
// New memory is zeroed with cudaMemset, which runs on the legacy default
// stream and is not ordered with the caller's stream if that stream was
// created non-blocking; the device is therefore synchronised after zeroing,
// so that no kernel on any stream can see the memory before it is zero.
int ensure_workspace(int dev, size_t ll_need, Workspace** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  Workspace& w = g_ws[dev];
  bool zeroed = false;
  if (!w.ctrl) {
    const size_t words = kCtrlWords + static_cast<size_t>(kPhases) * kSigPhaseWords;
    void* p = nullptr;
    if (cudaMalloc(&p, words * sizeof(uint32_t)) != cudaSuccess) {
      cudaGetLastError();
      return VRAR_ENOMEM;
    }
    if (cudaMemset(p, 0, words * sizeof(uint32_t)) != cudaSuccess) {
      cudaFree(p);
      return cuda_fail(cudaErrorUnknown);
    }
    zeroed = true;
    w.ctrl = static_cast<uint32_t*>(p);
    w.sig = w.ctrl + kCtrlWords;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return cuda_fail(cudaErrorUnknown);
    w.sms = sms;
  }
  if (ll_need > w.ll_bytes) {
    if (w.ll) {
      if (cudaDeviceSynchronize() != cudaSuccess) return cuda_fail(cudaErrorUnknown);
      cudaFree(w.ll);
      w.ll = nullptr;
      w.ll_bytes = 0;
    }
    const size_t bytes = (ll_need + (1u << 20) - 1) & ~static_cast<size_t>((1u << 20) - 1);
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
      cudaGetLastError();
      return VRAR_ENOMEM;
    }
    if (cudaMemset(p, 0, bytes) != cudaSuccess) {
      cudaFree(p);
      return cuda_fail(cudaErrorUnknown);
    }
    zeroed = true;
    w.ll = static_cast<uint64_t*>(p);
    w.ll_bytes = bytes;
  }
  if (zeroed && cudaDeviceSynchronize() != cudaSuccess) return cuda_fail(cudaErrorUnknown);
  *out = &w;
  return VRAR_OK;
}

// Status and failure info of the allocation-free entry point's control words
// on device `dev` (defined with that entry point below): reads them into
// h[kCtrlWords] and clears status and info on the device. *present is false
// when that entry point has not been set up on the device.
int noalloc_take_status(int dev, uint32_t* h, bool* present);

// ---- argument checks -------------------------------------------------------------------

struct Range {
  uintptr_t lo, hi;
};

bool overlap(const Range& a, const Range& b) { return a.lo < b.hi && b.lo < a.hi; }

int check_buffers(const void* const in[], void* const out[], int P, size_t in_elems, size_t out_elems,
                  vrar_dtype_t dt) {
  if (!in || !out) return VRAR_EINVAL;
  if (P < 1 || P > kMaxRanks) return VRAR_EINVAL;
  if (!valid_dtype(dt)) return VRAR_EINVAL;
  const size_t es = elem_size(dt);
  if (in_elems > (SIZE_MAX / 2) / es || out_elems > (SIZE_MAX / 2) / es) return VRAR_EINVAL;
  Range ri[kMaxRanks], ro[kMaxRanks];
  for (int p = 0; p < P; ++p) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(in[p]), b = reinterpret_cast<uintptr_t>(out[p]);
    if (!a || !b || (a & 15u) || (b & 15u)) return VRAR_EINVAL;
    ri[p] = {a, a + in_elems * es};
    ro[p] = {b, b + out_elems * es};
  }
  if (in_elems == 0 || out_elems == 0) return VRAR_OK;
  for (int q = 0; q < P; ++q) {
    for (int p = 0; p < P; ++p)
      if (overlap(ro[q], ri[p])) return VRAR_EINVAL;
    for (int p = q + 1; p < P; ++p)
      if (overlap(ro[q], ro[p])) return VRAR_EINVAL;
  }
  return VRAR_OK;
}

int check_shape(vrar_algo_t algo, int P, int L) {
  switch (algo) {
    case VRAR_ALGO_ONESHOT:
    case VRAR_ALGO_TWOSTAGE:
    case VRAR_ALGO_TWOSTAGE_WRITE:
      return VRAR_OK;
    case VRAR_ALGO_RD:
      return is_pow2(P) ? VRAR_OK : VRAR_ENOTSUP;
    case VRAR_ALGO_HIER:
      return (L >= 1 && P % L == 0 && is_pow2(P / L)) ? VRAR_OK : VRAR_ENOTSUP;
    default:
      return VRAR_EINVAL;
  }
}

// fp32 partials on the wire apply to recursive doubling and the hierarchical
// algorithm with 16-bit elements (for fp32 elements both wires are the same).
bool wide_wire(vrar_algo_t algo, vrar_dtype_t dt) {
  return g_set.payload_wire.load() == VRAR_WIRE_FP32 && dt != VRAR_FP32 &&
         (algo == VRAR_ALGO_RD || algo == VRAR_ALGO_HIER);
}

// Payload-slot bytes (RD / HIER) of a call whose grid covers the message in
// one round: P ranks x steps x items-per-slot x 32 bytes, twice that with fp32
// partials of 16-bit elements (two quads per item). A call that needs several
// rounds uses two slot sets of C x (threads per rank) slots instead, which is
// less than twice this; so twice this bounds every launch of the shape.
size_t one_round_slot_bytes(vrar_algo_t algo, int P, size_t n, vrar_dtype_t dt, int L) {
  const int64_t items = (static_cast<int64_t>(n) + per_item(dt) - 1) / per_item(dt);
  const size_t wide = wide_wire(algo, dt) ? 2 : 1;
  if (algo == VRAR_ALGO_RD) return wide * static_cast<size_t>(P) * ilog2(P) * items * 32;
  if (algo == VRAR_ALGO_HIER) {
    const int64_t piece = (items + L - 1) / L;
    return wide * static_cast<size_t>(P) * ilog2(P / L) * piece * 32;
  }
  return 0;
}

// SM count of a device (cached).
int device_sms(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  int v = cache[dev].load();
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1) {
    cudaGetLastError();
    return 0;
  }
  cache[dev] = v;
  return v;
}

// ---- launch -----------------------------------------------------------------------------

using KernelFn = void (*)(KArgs);

// Upper bound on CTAs per SM a call may use (0 = as many as fit). Leaving
// room lets the next call's CTAs become resident, and start their L2
// prefetches, while this call is still running.
#ifndef VRAR_CTAS_PER_SM
#define VRAR_CTAS_PER_SM 0
#endif

// Raise a kernel's dynamic shared-memory limit on the current device to at
// least `smem` bytes (never lowers it: an earlier, larger launch may rely on it).
bool ensure_smem_limit(KernelFn fn, int dev, size_t smem) {
  struct Entry {
    KernelFn fn;
    int dev;
    size_t limit;
  };
  static std::mutex mu;
  static Entry set[256];
  static int used = 0;
  // Set for any dynamic size: the 48 KiB default covers static shared memory
  // too, so a launch just under it can still be refused without the attribute.
  if (smem == 0) return true;
  std::lock_guard<std::mutex> lock(mu);
  Entry* e = nullptr;
  for (int i = 0; i < used; ++i)
    if (set[i].fn == fn && set[i].dev == dev) e = &set[i];
  if (e && e->limit >= smem) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (e) e->limit = smem;
  else if (used < 256) set[used++] = {fn, dev, smem};
  return true;
}

// CTAs resident per SM for a kernel with `threads` threads and `smem` bytes of
// dynamic shared memory (cached per kernel, device and smem size); 0 if the
// kernel cannot be given that much shared memory.
int resident_ctas(KernelFn fn, int dev, int sms, int threads = kThreads, size_t smem = 0) {
  struct Entry {
    KernelFn fn;
    int dev;
    size_t smem;
    int occ;
  };
  static std::mutex mu;
  static Entry cache[512];
  static int used = 0;
  if (!ensure_smem_limit(fn, dev, smem)) return 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].fn == fn && cache[i].dev == dev && cache[i].smem == smem) return cache[i].occ * sms;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, smem) != cudaSuccess || occ < 1) {
    cudaGetLastError();
    occ = 1;
  }
  if (VRAR_CTAS_PER_SM > 0 && occ > VRAR_CTAS_PER_SM) occ = VRAR_CTAS_PER_SM;
  if (used < 512) cache[used++] = {fn, dev, smem, occ};
  return occ * sms;
}

// The CTAs one call may use: what fits on the device at once, or fewer if the
// caller set a budget (vrar_set_max_ctas) to leave SMs to concurrent work.
int grid_budget(KernelFn fn, int dev, int sms, int threads = kThreads, size_t smem = 0) {
  const int resident = resident_ctas(fn, dev, sms, threads, smem);
  const int cap = g_set.max_ctas.load();
  return (cap > 0 && resident > cap) ? cap : resident;
}

// CTAs per rank: enough for one item per thread over `work_items` (the items
// one rank handles), at most what keeps the whole grid resident.
int blocks_per_rank(int64_t work_items, int P, int max_ctas, int threads = kThreads) {
  const int64_t want = std::max<int64_t>(1, (work_items + threads - 1) / threads);
  const int64_t cap = std::max(1, std::min(max_ctas, kMaxCtas) / P);
  return static_cast<int>(std::min(want, cap));
}

template <class D>
KernelFn pick_kernel(vrar_algo_t algo, int C) {
#define VRAR_CHUNK_CASES(K)          \
  switch (C) {                       \
    case 1: return K<D, 1>;          \
    case 2: return K<D, 2>;          \
    case 3: return K<D, 3>;          \
    case 4: return K<D, 4>;          \
    case 5: return K<D, 5>;          \
    case 6: return K<D, 6>;          \
    case 7: return K<D, 7>;          \
    default: return K<D, 8>;         \
  }
  switch (algo) {
    case VRAR_ALGO_ONESHOT: return k_oneshot<D>;
    case VRAR_ALGO_TWOSTAGE: return k_twostage<D>;
    case VRAR_ALGO_TWOSTAGE_WRITE: return k_twostage_write<D>;
    case VRAR_ALGO_RD: VRAR_CHUNK_CASES(k_rd)
    case VRAR_ALGO_HIER: VRAR_CHUNK_CASES(k_hier)
    default: return nullptr;
  }
#undef VRAR_CHUNK_CASES
}

// Programmatic dependent launch is on unless VRAR_PDL=0 (read once).
bool pdl_enabled() {
  static int cached = -1;
  if (cached < 0) {
    const char* s = std::getenv("VRAR_PDL");
    cached = (s && s[0] == '0') ? 0 : 1;
  }
  return cached == 1;
}

// Payload pieces each thread keeps in flight in the RD / HIER exchange: at
// most the configured C, but no more than it takes for the resident grid to
// cover a rank's `work` items in one round, so that a short message is spread
// over many threads instead of being stacked C deep on a few. Results do not
// depend on this choice.
template <class D>
int rd_chunks_for(vrar_algo_t algo, int C, int64_t work, int P, int dev, int sms) {
  for (int c = 1; c < C; ++c) {
    const int cap = std::max(1, std::min(grid_budget(pick_kernel<D>(algo, c), dev, sms), kMaxCtas) / P);
    if ((work + c - 1) / c <= static_cast<int64_t>(cap) * kThreads) return c;
  }
  return C;
}

int launch(KernelFn fn, const KArgs& a, int grid, cudaStream_t stream, int threads = kThreads, size_t smem = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fn, a);
  if (e != cudaSuccess) return cuda_fail(e);
  return VRAR_OK;
}

// Which write-mode kernel runs: VRAR_WRITE_KERNEL=plain|staged|async|batched
// forces one (read once); otherwise write_kernel_for() decides by shape.
enum WriteKernel { kWritePlain = 0, kWriteStaged = 1, kWriteAsync = 2, kWriteBatched = 3 };

int write_kernel_override() {
  static int cached = -2;
  if (cached == -2) {
    const char* s = std::getenv("VRAR_WRITE_KERNEL");
    cached = !s                               ? -1
             : std::strcmp(s, "plain") == 0  ? kWritePlain
             : std::strcmp(s, "staged") == 0 ? kWriteStaged
             : std::strcmp(s, "async") == 0  ? kWriteAsync
             : std::strcmp(s, "batched") == 0 ? kWriteBatched
                                             : -1;
  }
  return cached;
}

// Per-shape choice measured on a B200 (CUDA-graph timings of back-to-back
// calls, inputs rotated through more than 3x the L2 size): 'O' one-shot,
// 'A' write mode with the per-thread async-copy kernel, 'S' write mode with
// the bulk-copy staged kernel, 'P' write mode with the plain kernel, 'B'
// write mode with the register-batched kernel. Rows: P <= 2, 4, 8, 16, 32;
// columns: bytes per rank <= 32 KiB, 64 KiB, ..., 32 MiB, and above. One-shot
// keeps small messages at two and four ranks (one pass, its re-reads served by
// L2); at two and four ranks and 2 MiB per rank the batched write kernel is
// faster (2.27 against one-shot's 3.19 us at two ranks, 3.23 against the
// async kernel's 3.46 at four). The async write kernel wins almost everywhere
// else up to a few MiB: every thread keeps all P loads of its items in flight,
// with no serial issue. From 8 MiB per rank at 4-16 ranks the bulk-copy pipeline
// streams a little better. Past the L2-sized messages, where every byte comes
// from DRAM, the plain kernel (one 512-thread CTA per SM, eight loads per
// thread in flight, stores staggered by rank) streams best at eight ranks and
// more: 607.6 against 624.0 (batched), 638.3 (async) and 649.2 us (staged) at
// 8 x 224 MiB, 176.0 against 179.5, 188.0 and 190.0 at 8 x 64 MiB, 180.1
// against 186.9 (async) at 32 x 16 MiB. At two and four ranks a plain thread
// has only P loads in flight; there the batched kernel (two items per thread)
// is fastest above 16 MiB at four ranks (88.1 against 96.2 us at 64 MiB) and
// above 32 MiB at two.
constexpr int kChoiceCols = 12;
constexpr char kChoice[5][kChoiceCols] = {
    {'O', 'O', 'O', 'O', 'O', 'O', 'B', 'A', 'A', 'A', 'A', 'B'},  // P <= 2
    {'O', 'O', 'A', 'O', 'O', 'A', 'B', 'A', 'S', 'A', 'B', 'B'},  // P <= 4
    {'A', 'A', 'A', 'A', 'A', 'A', 'A', 'A', 'S', 'S', 'P', 'P'},  // P <= 8
    {'A', 'A', 'A', 'A', 'A', 'A', 'A', 'A', 'S', 'P', 'P', 'P'},  // P <= 16
    {'A', 'A', 'A', 'A', 'A', 'A', 'A', 'P', 'P', 'P', 'P', 'P'},  // P <= 32
};

// The write-mode kernel with fp8 payloads on, measured the same way (rows and
// columns as kChoice). With fp8 the kernels are bound by the quantisation
// arithmetic (P + 1 groups of 8 per item), not by memory, so what counts is
// the warps each SM keeps issuing. The async kernel wins small messages. Its
// shared-memory stages grow with P and cut its CTAs per SM, so from 512 KiB -
// 1 MiB per rank at 16 and 32 ranks the plain kernel's 512-thread CTAs win
// (at 32 ranks x 2 MiB: 62.2 against 133.1 us async; x 64 MiB: 1927 against 3711);
// at 4 ranks from 1 MiB the staged kernel (226 against 240 us async at
// 64 MiB); at 8 ranks the async kernel from 4 MiB (410 against 445 us plain at
// 64 MiB).
constexpr char kChoiceFp8[5][kChoiceCols] = {
    {'A', 'A', 'A', 'A', 'P', 'P', 'A', 'A', 'A', 'A', 'A', 'A'},  // P <= 2
    {'A', 'A', 'A', 'A', 'A', 'S', 'S', 'S', 'S', 'S', 'S', 'S'},  // P <= 4
    {'A', 'A', 'A', 'A', 'A', 'P', 'B', 'A', 'A', 'A', 'A', 'A'},  // P <= 8
    {'A', 'A', 'A', 'A', 'A', 'P', 'P', 'P', 'P', 'P', 'P', 'P'},  // P <= 16
    {'A', 'A', 'A', 'A', 'P', 'P', 'P', 'P', 'P', 'P', 'P', 'P'},  // P <= 32
};

char table_choice(const char (&table)[5][kChoiceCols], int P, size_t bytes) {
  const int row = P <= 2 ? 0 : P <= 4 ? 1 : P <= 8 ? 2 : P <= 16 ? 3 : 4;
  int col = 0;
  while (col < kChoiceCols - 1 && bytes > (static_cast<size_t>(32) << 10 << col)) ++col;
  return table[row][col];
}

char shape_choice(int P, size_t bytes) { return P <= 1 ? 'O' : table_choice(kChoice, P, bytes); }

// Which write-mode kernel runs a TWOSTAGE_WRITE call. Shapes the table gives
// to one-shot (when write mode is asked for by name) take the async kernel,
// the fastest write kernel on small messages. With fp8 payloads (q8) the
// kernel comes from kChoiceFp8; the algorithm AUTO runs does not depend on
// fp8 (one-shot and write mode pass different values through the fp8 wire, so
// the result stays a function of the shape alone).
int write_kernel_for(int P, size_t bytes, bool q8 = false) {
  const int forced = write_kernel_override();
  if (forced >= 0) return forced;
  const char ch = q8 ? table_choice(kChoiceFp8, P, bytes) : shape_choice(P, bytes);
  return ch == 'P' ? kWritePlain : ch == 'S' ? kWriteStaged : ch == 'B' ? kWriteBatched : kWriteAsync;
}

// Async-copy kernel: 64 items (one per thread) per tile, and S tiles in flight
// per thread. S is set from the bytes a CTA should keep in flight, measured:
// small messages give each CTA only a tile or two, and they run fastest with
// deep stages (about 192 KiB per CTA up to 64 KiB per rank, 96 KiB up to
// 256 KiB); from 512 KiB per rank smaller CTAs, more of them per SM, do better
// (48 KiB, then 32 KiB). With a CTA budget of at most one CTA per SM every CTA
// keeps the deepest setting. S is rounded down to an instantiated depth
// (3, 4, 6 or 8).
constexpr int kAsyncTileItems = 64;

int async_stages(int P, size_t bytes_per_rank, bool deep) {
  const size_t kib = 1024;
  const size_t target = deep || bytes_per_rank <= 64 * kib ? 192 * kib
                        : bytes_per_rank <= 256 * kib      ? 96 * kib
                        : bytes_per_rank <= 512 * kib      ? 48 * kib
                                                           : 32 * kib;
  const size_t s = target / (static_cast<size_t>(P) * kAsyncTileItems * 16);
  return s >= 8 ? 8 : s >= 6 ? 6 : s >= 4 ? 4 : 3;
}

// One-shot on small messages (at most 1 MiB of input over all P ranks):
// 128-thread CTAs, more of them, measured faster there (1.46 vs 1.60 us at
// 2 ranks x 128 KiB, 2.37 vs 2.64 us at 8 x 128 KiB); above it the 512-thread
// CTAs are faster (2.62 vs 3.59 us at 8 x 256 KiB, 4.06 vs 5.86 at 16 x 128 KiB).
constexpr size_t kOneshotSmallBytes = 1 << 20;
constexpr size_t kRsAsyncMaxBytes = 1 << 20;  // reduce-scatter: async scatter form up to here (bytes per rank)
constexpr int kSmallThreads = 128;

// The pull 2-stage with 256-thread CTAs: more, smaller CTAs share each column's
// mid barrier (measured 6-10 % faster than 512 from 128 KiB to 2 MiB per rank).
constexpr int kPullThreads = 256;

// The plain write kernel budgets its registers for one 512-thread CTA per SM,
// which streams DRAM-sized calls best (608 against 638 us with two at
// 8 x 224 MiB, 180 against 199 us at 32 x 16 MiB, 48.3 against 49.5 us at
// 32 x 4 MiB). A call that moves at most this many bytes (2 P n s) and that one
// CTA per SM cannot cover in one pass takes the two-CTA build instead (at 2 ranks
// x 2 MiB: 256 CTAs in one pass, 2.36 against 3.60 us; x 4 MiB: 4.62 against
// 6.39 us); one that fits in one pass keeps one CTA per SM (2 x 1 MiB: 2.03
// against 2.51 us).
constexpr size_t kPlainTwoPerSmBytes = 32u << 20;

// Above that size the one-CTA build runs on at most this many CTAs: fewer
// concurrent streams draw more from DRAM (at 8 x 224 MiB: 608.5 against 620.4
// us with 144 CTAs; 16 x 64 MiB: 343.1 against 348.9; 16 x 32 MiB: 171.7
// against 174.5; 112 CTAs are slower again: 643.8 us at 8 x 224 MiB).
constexpr int kPlainDramCtas = 128;

// Kernels of the custom all-reduce (one-shot, pull 2-stage, plain write), with
// or without the fp8 wire (q8, 16-bit element types only; the host rejects
// fp8 for fp32 before it gets here). two_per_sm picks the plain write kernel's
// two-CTA budget (not with q8).
template <class D>
KernelFn custom_kernel(vrar_algo_t algo, int threads, bool q8, bool two_per_sm = false) {
  if constexpr (D::VE == 8) {
    if (q8) {
      if (algo == VRAR_ALGO_ONESHOT)
        return threads == kSmallThreads ? k_oneshot<D, kSmallThreads, true> : k_oneshot<D, kThreads, true>;
      if (algo == VRAR_ALGO_TWOSTAGE) return k_twostage<D, kPullThreads, true>;
      return k_twostage_write<D, true>;
    }
  }
  if (algo == VRAR_ALGO_ONESHOT) return threads == kSmallThreads ? k_oneshot<D, kSmallThreads> : k_oneshot<D>;
  if (algo == VRAR_ALGO_TWOSTAGE) return k_twostage<D, kPullThreads>;
  return two_per_sm ? k_twostage_write<D, false, 2> : k_twostage_write<D>;
}

KernelFn custom_kernel_dt(vrar_dtype_t dt, vrar_algo_t algo, int threads, bool q8, bool two_per_sm = false) {
  return dt == VRAR_BF16   ? custom_kernel<Bf16T>(algo, threads, q8, two_per_sm)
         : dt == VRAR_FP16 ? custom_kernel<F16T>(algo, threads, q8, two_per_sm)
                           : custom_kernel<F32T>(algo, threads, false, two_per_sm);
}

// HIER (element wire) by size, measured at 4 groups x 8 ranks: up to 256 KiB
// per rank one 512-thread CTA per SM (7.8 vs 9.9 us; the call is one round
// over its items and the 64-register build spills); above it two CTAs per SM
// (43 vs 50 us at 2 MiB with one piece per thread, 204 vs 226 us at 8 MiB
// with two).
constexpr size_t kHierOneCtaBytes = 256 << 10;
constexpr size_t kHierOnePieceBytes = 2 << 20;

// HIER warms L2 with each next round's group inputs up to 2 MiB per rank
// (measured: 18.7 against 20.1 us at 4 x 8 ranks x 1 MiB, 16.3 against 17.8 at
// 2 x 8 x 2 MiB, 20.5 against 22.2 at 4 x 2 x 2 MiB); above it the early loads
// evict payload slots (209 against 177 us at 4 x 8 x 8 MiB).
constexpr size_t kHierPrefetchBytes = 2 << 20;

template <class D>
KernelFn hier_two_per_sm(int C) {
  return C <= 1 ? k_hier<D, 1, 2> : k_hier<D, 2, 2>;
}

// Recursive doubling on the element wire: two 512-thread CTAs per SM with at
// most two payload pieces per thread (64 registers, no spills). Measured at 8
// ranks with 256-bit payload accesses, graphs of 200 calls: 8.67 / 15.2 / 28.8
// / 97.0 us at 512 KiB / 1 / 2 / 8 MiB per rank, against 9.29 / 16.0 / 29.6 /
// 105.3 us with one CTA per SM and four pieces (more pieces in the two-CTA
// build spill: 57 us at 2 MiB with four).
template <class D>
KernelFn rd_two_per_sm(int C) {
  return C <= 1 ? k_rd<D, 1, 2> : k_rd<D, 2, 2>;
}

KernelFn rd_two_per_sm_dt(vrar_dtype_t dt, int C) {
  return dt == VRAR_BF16 ? rd_two_per_sm<Bf16T>(C) : dt == VRAR_FP16 ? rd_two_per_sm<F16T>(C)
                                                                    : rd_two_per_sm<F32T>(C);
}

KernelFn hier_two_per_sm_dt(vrar_dtype_t dt, int C) {
  return dt == VRAR_BF16 ? hier_two_per_sm<Bf16T>(C) : dt == VRAR_FP16 ? hier_two_per_sm<F16T>(C)
                                                                      : hier_two_per_sm<F32T>(C);
}

template <class D>
KernelFn async_rs_kernel(int S) {
  switch (S) {
    case 8: return k_twostage_write_async<D, kAsyncTileItems, 8, true>;
    case 6: return k_twostage_write_async<D, kAsyncTileItems, 6, true>;
    case 4: return k_twostage_write_async<D, kAsyncTileItems, 4, true>;
    default: return k_twostage_write_async<D, kAsyncTileItems, 3, true>;
  }
}

KernelFn async_rs_kernel_dt(vrar_dtype_t dt, int S) {
  return dt == VRAR_BF16 ? async_rs_kernel<Bf16T>(S) : dt == VRAR_FP16 ? async_rs_kernel<F16T>(S)
                                                                     : async_rs_kernel<F32T>(S);
}

template <class D, bool Q>
KernelFn async_kernel(int S) {
  switch (S) {
    case 8: return k_twostage_write_async<D, kAsyncTileItems, 8, false, Q>;
    case 6: return k_twostage_write_async<D, kAsyncTileItems, 6, false, Q>;
    case 4: return k_twostage_write_async<D, kAsyncTileItems, 4, false, Q>;
    default: return k_twostage_write_async<D, kAsyncTileItems, 3, false, Q>;
  }
}

KernelFn async_kernel_dt(vrar_dtype_t dt, int S, bool q8) {
  if (dt == VRAR_BF16) return q8 ? async_kernel<Bf16T, true>(S) : async_kernel<Bf16T, false>(S);
  if (dt == VRAR_FP16) return q8 ? async_kernel<F16T, true>(S) : async_kernel<F16T, false>(S);
  return async_kernel<F32T, false>(S);
}

// Staged write mode without a CTA budget: items per tile (64: 1 KiB per input
// rank), the shared-memory bytes of stages a CTA aims for, and the most stages.
#ifndef VRAR_STAGED_TILE
#define VRAR_STAGED_TILE 64
#endif
#ifndef VRAR_STAGED_BYTES
#define VRAR_STAGED_BYTES (96 * 1024)
#endif
#ifndef VRAR_STAGED_MAX_STAGES
#define VRAR_STAGED_MAX_STAGES 6
#endif
constexpr int kWriteTileItems = VRAR_STAGED_TILE;
static_assert(kWriteTileItems == 64 || kWriteTileItems == 128, "staged tiles of 64 or 128 items are instantiated");

template <class D, bool Q>
KernelFn staged_kernel(int ti) {
  return ti == 64 ? k_twostage_write_staged<D, 64, Q> : k_twostage_write_staged<D, 128, Q>;
}

// Dispatch on the element type.
KernelFn pick_kernel_dt(vrar_dtype_t dt, vrar_algo_t algo, int C) {
  return dt == VRAR_BF16 ? pick_kernel<Bf16T>(algo, C) : dt == VRAR_FP16 ? pick_kernel<F16T>(algo, C)
                                                                        : pick_kernel<F32T>(algo, C);
}

// Items each thread of the batched write kernel keeps in flight per input rank.
#ifndef VRAR_BATCH_ITEMS
#define VRAR_BATCH_ITEMS 2
#endif

template <class D, bool Q>
KernelFn batched_kernel(int P) {
  return P <= 8    ? k_twostage_write_batched<D, VRAR_BATCH_ITEMS, 8, Q>
         : P <= 16 ? k_twostage_write_batched<D, VRAR_BATCH_ITEMS, 16, Q>
                   : k_twostage_write_batched<D, VRAR_BATCH_ITEMS, 32, Q>;
}

KernelFn batched_kernel_dt(vrar_dtype_t dt, int P, bool q8) {
  if (dt == VRAR_BF16) return q8 ? batched_kernel<Bf16T, true>(P) : batched_kernel<Bf16T, false>(P);
  if (dt == VRAR_FP16) return q8 ? batched_kernel<F16T, true>(P) : batched_kernel<F16T, false>(P);
  return batched_kernel<F32T, false>(P);
}

KernelFn staged_kernel_dt(vrar_dtype_t dt, int ti, bool q8) {
  if (dt == VRAR_BF16) return q8 ? staged_kernel<Bf16T, true>(ti) : staged_kernel<Bf16T, false>(ti);
  if (dt == VRAR_FP16) return q8 ? staged_kernel<F16T, true>(ti) : staged_kernel<F16T, false>(ti);
  return staged_kernel<F32T, false>(ti);
}

// fp32 partials on the wire. RD runs two CTAs per SM with one piece per thread
// (measured at 8 ranks: 30.6 / 51.6 / 196 us at 1 / 2 / 8 MiB per rank against
// 31.4 / 57.6 / 205 us with one CTA per SM and two pieces; two pieces in the
// two-CTA build spill). HIER keeps one CTA per SM (47.0 against 57.8 us at
// 4 x 8 ranks x 2 MiB with two).
template <class D>
KernelFn pick_wide(vrar_algo_t algo, int C) {
  if (algo == VRAR_ALGO_RD) return k_rd_wide<D, 1, 2>;
  return C <= 1 ? k_hier_wide<D, 1> : k_hier_wide<D, 2>;
}

KernelFn pick_wide_dt(vrar_dtype_t dt, vrar_algo_t algo, int C) {
  return dt == VRAR_BF16 ? pick_wide<Bf16T>(algo, C) : pick_wide<F16T>(algo, C);
}

// Chunk count for the fp32-wire kernels (at most 2, see k_rd_wide; RD takes 1,
// see pick_wide), chosen like rd_chunks_for.
int wide_chunks_for(vrar_dtype_t dt, vrar_algo_t algo, int C, int64_t work, int P, int dev, int sms) {
  C = algo == VRAR_ALGO_RD ? 1 : std::min(C, 2);
  for (int c = 1; c < C; ++c) {
    const int cap = std::max(1, std::min(grid_budget(pick_wide_dt(dt, algo, c), dev, sms), kMaxCtas) / P);
    if ((work + c - 1) / c <= static_cast<int64_t>(cap) * kThreads) return c;
  }
  return C;
}

int rd_chunks_for_dt(vrar_dtype_t dt, vrar_algo_t algo, int C, int64_t work, int P, int dev, int sms) {
  return dt == VRAR_BF16   ? rd_chunks_for<Bf16T>(algo, C, work, P, dev, sms)
         : dt == VRAR_FP16 ? rd_chunks_for<F16T>(algo, C, work, P, dev, sms)
                           : rd_chunks_for<F32T>(algo, C, work, P, dev, sms);
}

// The launch of a recursive-doubling or hierarchical call and the payload
// slots it uses (the layout is described with k_rd in kernels.cuh).
struct PayloadPlan {
  KernelFn fn = nullptr;
  int C = 1;                 // payload pieces per thread
  int B = 1;                 // CTAs per rank
  int64_t slot_items = 0;    // 32-byte slots per rank, step and slot set
  int slot_sets = 1;         // 1: one round, slot = item index; 2: slots reused by round parity
  size_t bytes = 0;          // slot bytes in all: slot_sets * P * steps * slot_items * 32
};

// Whether a kernel uses local memory (register spills or a stack frame). The
// CUDA driver reserves local memory for the whole device the first time it
// runs a kernel that needs some, which is an allocation the allocation-free
// entry point avoids by preferring kernels that need none. Cached per kernel.
bool uses_local_memory(KernelFn fn) {
  static std::mutex mu;
  static KernelFn seen[256];
  static bool local[256];
  static int used = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (seen[i] == fn) return local[i];
  cudaFuncAttributes at;
  bool v = true;
  if (cudaFuncGetAttributes(&at, fn) == cudaSuccess) v = at.localSizeBytes > 0;
  else cudaGetLastError();
  if (used < 256) {
    seen[used] = fn;
    local[used++] = v;
  }
  return v;
}

// C_cfg: the configured chunk count. `fit_one_round` (the allocation-free
// entry point) takes the smallest chunk count up to the kernels' maximum that
// covers the message in one round, whatever C_cfg is; if none does, at most 4
// (at most 1 on the fp32 wire), and few enough CTAs per rank that its two slot
// sets stay within the one-round size. Among those it skips kernels that use
// local memory when a larger (or, past one round, smaller) chunk count gives
// one that uses none.
int plan_payload(vrar_algo_t algo, int P, size_t n, vrar_dtype_t dt, int L, int dev, int sms, int C_cfg,
                 bool fit_one_round, PayloadPlan* out) {
  PayloadPlan pl;
  const bool wide = wide_wire(algo, dt);
  const int64_t items = (static_cast<int64_t>(n) + per_item(dt) - 1) / per_item(dt);
  const int64_t piece = algo == VRAR_ALGO_RD ? items : (items + L - 1) / L;  // items one rank exchanges
  const int steps = algo == VRAR_ALGO_RD ? ilog2(P) : ilog2(P / L);
  int C = std::min(8, std::max(1, C_cfg));
  // HIER keeps one payload piece per thread up to 2 MiB per rank and at most
  // two above: its in-group phases already keep L loads and L stores per
  // piece in flight, and more pieces cost registers (measured, 4 groups x 8,
  // both wires; e.g. 226 vs 251 us at 8 MiB, two pieces against four, and
  // 78 vs 84 us at 2 MiB with fp32 partials, one against two). Above 256 KiB
  // per rank the element-wire kernel also runs two CTAs per SM (below).
  if (algo == VRAR_ALGO_HIER) C = n * elem_size(dt) <= kHierOnePieceBytes ? 1 : std::min(C, 2);
  if (fit_one_round) {
    auto kern = [&](int c) { return wide ? pick_wide_dt(dt, algo, c) : pick_kernel_dt(dt, algo, c); };
    const int cmax = wide ? (algo == VRAR_ALGO_RD ? 1 : 2) : 8;  // the kernels' largest chunk count
    int pick = 0, pick_any = 0;
    for (int c = 1; c <= cmax && !pick; ++c) {
      const int cap = std::max(1, std::min(grid_budget(kern(c), dev, sms), kMaxCtas) / P);
      if ((piece + c - 1) / c <= static_cast<int64_t>(cap) * kThreads) {
        if (!pick_any) pick_any = c;
        if (!uses_local_memory(kern(c))) pick = c;
      }
    }
    if (!pick) pick = pick_any;
    if (!pick) {  // several rounds: at most 4 pieces (1 on the fp32 wire), preferring no local memory
      const int top = wide ? 1 : std::min(C, 4);
      for (int c = top; c >= 1 && !pick; --c)
        if (!uses_local_memory(kern(c))) pick = c;
      if (!pick) pick = top;
    }
    C = pick;
  } else if (algo == VRAR_ALGO_RD && !wide) {
    // Two CTAs per SM, at most two pieces: the fewest pieces that cover the
    // message in one round with that grid, else two.
    C = std::min(C, 2);
    const int cap = std::max(1, std::min(grid_budget(rd_two_per_sm_dt(dt, 1), dev, sms), kMaxCtas) / P);
    if (C > 1 && piece <= static_cast<int64_t>(cap) * kThreads) C = 1;
  } else {
    C = wide ? wide_chunks_for(dt, algo, C, piece, P, dev, sms) : rd_chunks_for_dt(dt, algo, C, piece, P, dev, sms);
  }
  pl.C = C;
  pl.fn = wide ? pick_wide_dt(dt, algo, C) : pick_kernel_dt(dt, algo, C);
  if (algo == VRAR_ALGO_HIER && !wide && n * elem_size(dt) > kHierOneCtaBytes) pl.fn = hier_two_per_sm_dt(dt, C);
  if (algo == VRAR_ALGO_RD && !wide && !fit_one_round) pl.fn = rd_two_per_sm_dt(dt, C);
  if (!pl.fn) return VRAR_EINVAL;
  const int64_t per_chunk = (piece + C - 1) / C;
  pl.B = blocks_per_rank(per_chunk, P, grid_budget(pl.fn, dev, sms));
  if (fit_one_round && per_chunk > static_cast<int64_t>(pl.B) * kThreads) {
    // Several rounds: two slot sets of C * B * T slots each. Keep them within
    // the one-round size (piece slots), which is what the caller's limit is
    // stated in: B <= piece / (2 C T).
    const int64_t cap_b = std::max<int64_t>(1, piece / (2 * static_cast<int64_t>(C) * kThreads));
    if (pl.B > cap_b) pl.B = static_cast<int>(cap_b);
  }
  {
    // Even rounds: the fewest CTAs per rank that keep the round count at its
    // minimum, so that no round runs partly empty while every round pays the
    // full chain of exchanges (measured: RD at 8 ranks x 2 MiB 27.5 against
    // 29.0 us, 32 CTAs per rank against 37; HIER at 4 x 8 ranks x 2 MiB 34.8
    // against 38.5 us, 8 against 9).
    const int64_t stride0 = static_cast<int64_t>(pl.B) * kThreads;
    const int64_t r0 = (per_chunk + stride0 - 1) / stride0;
    if (r0 > 1) pl.B = static_cast<int>((per_chunk + r0 * kThreads - 1) / (r0 * kThreads));
  }
  const int64_t stride = static_cast<int64_t>(pl.B) * kThreads;
  const int64_t rounds = (per_chunk + stride - 1) / stride;
  pl.slot_sets = rounds > 1 ? 2 : 1;
  pl.slot_items = (rounds > 1 ? static_cast<int64_t>(C) * stride : piece) * (wide ? 2 : 1);
  pl.bytes = static_cast<size_t>(pl.slot_sets) * P * steps * pl.slot_items * 32;
  *out = pl;
  return VRAR_OK;
}

const char* algo_name(int a) {
  switch (a) {
    case VRAR_ALGO_ONESHOT: return "oneshot";
    case VRAR_ALGO_TWOSTAGE: return "twostage";
    case VRAR_ALGO_TWOSTAGE_WRITE: return "twostage_write";
    case VRAR_ALGO_RD: return "rd";
    case VRAR_ALGO_HIER: return "hier";
    default: return "auto";
  }
}

// VRAR_ALGO from the environment (read once): forces the AUTO choice.
int env_algo() {
  static int cached = -2;
  if (cached != -2) return cached;
  int v = -1;
  if (const char* s = std::getenv("VRAR_ALGO")) {
    for (int a = VRAR_ALGO_ONESHOT; a <= VRAR_ALGO_HIER; ++a)
      if (std::strcmp(s, algo_name(a)) == 0) v = a;
  }
  cached = v;
  return v;
}

// The algorithm VRAR_ALGO_AUTO runs: one-shot or write mode per the measured
// table above. Recursive doubling and the hierarchical algorithm move 2x the
// data as payload words and never win on one device.
int select_algo(int P, size_t n, vrar_dtype_t dt) {
  return shape_choice(P, n * elem_size(dt)) == 'O' ? VRAR_ALGO_ONESHOT : VRAR_ALGO_TWOSTAGE_WRITE;
}

}  // namespace
}  // namespace vrar

using namespace vrar;

extern "C" {

int vrar_allreduce(const void* const rank_in[], void* const rank_out[], int P, size_t n, vrar_dtype_t dtype,
                   vrar_algo_t algo, vrar_stream_t stream) {
  int rc = check_buffers(rank_in, rank_out, P, n, n, dtype);
  if (rc != VRAR_OK) return rc;
  if (algo == VRAR_ALGO_AUTO) {
    const int forced = env_algo();
    algo = static_cast<vrar_algo_t>(forced > 0 ? forced : select_algo(P, n, dtype));
  }
  const int L = g_set.group_size.load();
  if ((rc = check_shape(algo, P, L)) != VRAR_OK) return rc;
  // fp8 payloads are defined for the custom all-reduce algorithms on 16-bit
  // elements (groups of 8 elements = one 16-byte item).
  const bool q8 = g_set.fp8_quant.load() != 0;
  if (q8 && (dtype == VRAR_FP32 || algo == VRAR_ALGO_RD || algo == VRAR_ALGO_HIER)) return VRAR_ENOTSUP;
  if (n == 0) return VRAR_OK;

  int dev = 0;
  if ((rc = current_device(&dev)) != VRAR_OK) return rc;
  const int sms = device_sms(dev);
  if (sms < 1) return VRAR_ECUDA;
  const bool payload = algo == VRAR_ALGO_RD || algo == VRAR_ALGO_HIER;
  PayloadPlan plan;
  if (payload && (rc = plan_payload(algo, P, n, dtype, L, dev, sms, g_set.rd_chunks.load(), false, &plan)) != VRAR_OK)
    return rc;
  Workspace* ws = nullptr;
  if ((rc = ensure_workspace(dev, payload ? plan.bytes : 0, &ws)) != VRAR_OK) return rc;
  const int C = payload ? plan.C : 1;
  KernelFn fn = payload ? plan.fn : pick_kernel_dt(dtype, algo, 1);
  if (!fn) return VRAR_EINVAL;

  KArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int p = 0; p < P; ++p) {
    a.ptr.in[p] = rank_in[p];
    a.ptr.out[p] = rank_out[p];
  }
  a.n = static_cast<int64_t>(n);
  a.items = (a.n + per_item(dtype) - 1) / per_item(dtype);
  a.P = P;
  a.L = L;
  a.chunks = C;
  a.edge_sync = g_set.edge_sync.load();
  a.fault_mask = g_set.fault_mask.load();
  a.timeout_ns = g_set.timeout_ns.load();
  a.ctrl = ws->ctrl;
  a.sig = ws->sig;
  a.ll = ws->ll;
  a.slot_items = plan.slot_items;
  a.slot_sets = plan.slot_sets;
  a.stats = g_set.spin_stats.load() ? reinterpret_cast<unsigned long long*>(ws->ctrl + kStats) : nullptr;
  if (payload) {
    a.steps = algo == VRAR_ALGO_RD ? ilog2(P) : ilog2(P / L);
    a.B = plan.B;
    a.prefetch_next = algo == VRAR_ALGO_HIER && n * elem_size(dtype) <= kHierPrefetchBytes;
    return launch(plan.fn, a, a.B * P, reinterpret_cast<cudaStream_t>(stream));
  }

  int64_t work = a.items;  // items one rank handles in its main loop
  switch (algo) {
    case VRAR_ALGO_ONESHOT: work = a.items; break;
    case VRAR_ALGO_TWOSTAGE:
    case VRAR_ALGO_TWOSTAGE_WRITE: work = (a.items + P - 1) / P; break;
    default: break;
  }
  const int wk = algo == VRAR_ALGO_TWOSTAGE_WRITE ? write_kernel_for(P, n * elem_size(dtype), q8) : kWritePlain;
  if (wk == kWriteAsync) {
    const int cap_budget = g_set.max_ctas.load();
    const bool deep = cap_budget > 0 && cap_budget <= sms;
    const int S = async_stages(P, n * elem_size(dtype), deep);
    KernelFn af = async_kernel_dt(dtype, S, q8);
    const int64_t tiles = std::max<int64_t>(1, (work + kAsyncTileItems - 1) / kAsyncTileItems);
    const size_t smem = static_cast<size_t>(S) * P * kAsyncTileItems * 16;
    const int resident = grid_budget(af, dev, sms, kAsyncTileItems, smem);
    if (resident < 1) return VRAR_ECUDA;
    a.B = static_cast<int>(std::min<int64_t>(tiles, std::max(1, std::min(resident, kMaxCtas) / P)));
    return launch(af, a, a.B * P, reinterpret_cast<cudaStream_t>(stream), kAsyncTileItems, smem);
  }
  if (wk == kWriteStaged) {
    // Normally 64-item tiles and about 96 KiB of stages per CTA (two CTAs per
    // SM). When a CTA budget leaves at most one CTA per SM, each CTA must keep
    // far more bytes in flight to draw its share of memory bandwidth: 128-item
    // tiles and up to 192 KiB of stages.
    const int cap_budget = g_set.max_ctas.load();
    const bool deep = cap_budget > 0 && cap_budget <= sms;
    const int ti = deep ? 128 : kWriteTileItems;
    KernelFn sf = staged_kernel_dt(dtype, ti, q8);
    const int64_t tiles = std::max<int64_t>(1, (work + ti - 1) / ti);
    const int S = std::max(2, std::min(deep ? kMaxStages : VRAR_STAGED_MAX_STAGES,
                                       (deep ? 192 * 1024 : VRAR_STAGED_BYTES) / (P * ti * 16)));
    const size_t smem = kStagedHeader + static_cast<size_t>(S) * P * ti * 16;
    const int resident = grid_budget(sf, dev, sms, 32 + ti, smem);
    const int B = static_cast<int>(std::min<int64_t>(tiles, std::max(1, std::min(resident, kMaxCtas) / P)));
    if (resident < 1) return VRAR_ECUDA;
    a.stages = S;
    a.B = B;
    return launch(sf, a, a.B * P, reinterpret_cast<cudaStream_t>(stream), 32 + ti, smem);
  }
  if (wk == kWriteBatched) {
    KernelFn bf = batched_kernel_dt(dtype, P, q8);
    const int64_t passes = std::max<int64_t>(1, (work + kBatchThreads * VRAR_BATCH_ITEMS - 1) /
                                                    (kBatchThreads * VRAR_BATCH_ITEMS));
    const int resident = grid_budget(bf, dev, sms, kBatchThreads);
    if (resident < 1) return VRAR_ECUDA;
    a.B = static_cast<int>(std::min<int64_t>(passes, std::max(1, std::min(resident, kMaxCtas) / P)));
    return launch(bf, a, a.B * P, reinterpret_cast<cudaStream_t>(stream), kBatchThreads);
  }
  int threads = kThreads;
  if (algo == VRAR_ALGO_ONESHOT && static_cast<size_t>(P) * n * elem_size(dtype) <= kOneshotSmallBytes)
    threads = kSmallThreads;
  if (algo == VRAR_ALGO_TWOSTAGE) threads = kPullThreads;
  fn = custom_kernel_dt(dtype, algo, threads, q8);
  int budget = grid_budget(fn, dev, sms, threads);
  const size_t call_bytes = 2 * static_cast<size_t>(P) * n * elem_size(dtype);
  if (algo == VRAR_ALGO_TWOSTAGE_WRITE && !q8 && call_bytes <= kPlainTwoPerSmBytes &&
      work > static_cast<int64_t>(std::min(budget, kMaxCtas) / P) * threads) {
    fn = custom_kernel_dt(dtype, algo, threads, false, true);  // one pass needs two CTAs per SM
    budget = grid_budget(fn, dev, sms, threads);
  } else if (algo == VRAR_ALGO_TWOSTAGE_WRITE && !q8 && call_bytes > kPlainTwoPerSmBytes) {
    budget = std::min(budget, kPlainDramCtas);
  }
  a.B = blocks_per_rank(work, P, budget, threads);
  return launch(fn, a, a.B * P, reinterpret_cast<cudaStream_t>(stream), threads);
}

int vrar_reduce_scatter(const void* const rank_in[], void* const rank_out[], int P, size_t n, vrar_dtype_t dtype,
                        vrar_stream_t stream) {
  if (P < 1 || P > kMaxRanks) return VRAR_EINVAL;
  if (n % static_cast<size_t>(P) != 0) return VRAR_EINVAL;
  int rc = check_buffers(rank_in, rank_out, P, n, n / P, dtype);
  if (rc != VRAR_OK) return rc;
  if (n == 0) return VRAR_OK;
  int dev = 0;
  if ((rc = current_device(&dev)) != VRAR_OK) return rc;
  const int sms = device_sms(dev);
  if (sms < 1) return VRAR_ECUDA;
  Workspace* ws = nullptr;
  if ((rc = ensure_workspace(dev, 0, &ws)) != VRAR_OK) return rc;
  KernelFn fn = dtype == VRAR_BF16   ? k_reduce_scatter<Bf16T>
                : dtype == VRAR_FP16 ? k_reduce_scatter<F16T>
                                     : k_reduce_scatter<F32T>;
  KArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int p = 0; p < P; ++p) {
    a.ptr.in[p] = rank_in[p];
    a.ptr.out[p] = rank_out[p];
  }
  a.n = static_cast<int64_t>(n);
  a.P = P;
  const int64_t m = a.n / P;
  if (m % per_item(dtype) == 0 && n * elem_size(dtype) <= kRsAsyncMaxBytes) {
    // Chunks of whole items: the async-copy kernel in scatter form (rank r's
    // slice of the write mode is exactly chunk r; the result goes to out[r]).
    // Measured faster up to 1 MiB per rank (3.0 vs 6.2 us at 32 x 256 KiB),
    // slower above it (3.9 vs 3.4 us at 8 x 2 MiB), where the plain kernel's
    // 512-thread CTAs keep more loads in flight for the single store.
    const int64_t mi = m / per_item(dtype);
    a.items = mi * P;
    const int cap_budget = g_set.max_ctas.load();
    const int S = async_stages(P, n * elem_size(dtype), cap_budget > 0 && cap_budget <= sms);
    KernelFn af = async_rs_kernel_dt(dtype, S);
    const int64_t tiles = std::max<int64_t>(1, (mi + kAsyncTileItems - 1) / kAsyncTileItems);
    const size_t smem = static_cast<size_t>(S) * P * kAsyncTileItems * 16;
    const int resident = grid_budget(af, dev, sms, kAsyncTileItems, smem);
    if (resident < 1) return VRAR_ECUDA;
    a.B = static_cast<int>(std::min<int64_t>(tiles, std::max(1, std::min(resident, kMaxCtas) / P)));
    return launch(af, a, a.B * P, reinterpret_cast<cudaStream_t>(stream), kAsyncTileItems, smem);
  }
  const int64_t work = (m % per_item(dtype) == 0) ? m / per_item(dtype) : m;
  a.B = blocks_per_rank(work, P, grid_budget(fn, dev, sms));
  return launch(fn, a, a.B * P, reinterpret_cast<cudaStream_t>(stream));
}

int vrar_all_gather(const void* const rank_in[], void* const rank_out[], int P, size_t n, vrar_dtype_t dtype,
                    vrar_stream_t stream) {
  if (P < 1 || P > kMaxRanks) return VRAR_EINVAL;
  if (n % static_cast<size_t>(P) != 0) return VRAR_EINVAL;
  int rc = check_buffers(rank_in, rank_out, P, n / P, n, dtype);
  if (rc != VRAR_OK) return rc;
  if (n == 0) return VRAR_OK;
  int dev = 0;
  if ((rc = current_device(&dev)) != VRAR_OK) return rc;
  const int sms = device_sms(dev);
  if (sms < 1) return VRAR_ECUDA;
  Workspace* ws = nullptr;
  if ((rc = ensure_workspace(dev, 0, &ws)) != VRAR_OK) return rc;
  KernelFn fn = dtype == VRAR_BF16   ? k_all_gather<Bf16T>
                : dtype == VRAR_FP16 ? k_all_gather<F16T>
                                     : k_all_gather<F32T>;
  KArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int p = 0; p < P; ++p) {
    a.ptr.in[p] = rank_in[p];
    a.ptr.out[p] = rank_out[p];
  }
  a.n = static_cast<int64_t>(n);
  a.P = P;
  const int64_t m = a.n / P;
  const int64_t work = (m % per_item(dtype) == 0) ? m / per_item(dtype) : m;
  const int budget = grid_budget(fn, dev, sms);
  a.B = blocks_per_rank(work, P, budget);
  // Destination groups: fill the resident grid when the slices are short.
  a.chunks = std::max(1, std::min(P, budget / (a.B * P)));
  return launch(fn, a, a.B * P * a.chunks, reinterpret_cast<cudaStream_t>(stream));
}

int vrar_select_algo(int P, size_t n, vrar_dtype_t dtype) {
  if (P < 1 || P > kMaxRanks || !valid_dtype(dtype)) return VRAR_EINVAL;
  return select_algo(P, n, dtype);
}

const char* vrar_kernel_name(int P, size_t n, vrar_dtype_t dtype, vrar_algo_t algo) {
  if (P < 1 || P > kMaxRanks || !valid_dtype(dtype) || algo < VRAR_ALGO_AUTO || algo > VRAR_ALGO_HIER)
    return nullptr;
  if (algo == VRAR_ALGO_AUTO) {
    const int forced = env_algo();
    algo = static_cast<vrar_algo_t>(forced > 0 ? forced : select_algo(P, n, dtype));
  }
  switch (algo) {
    case VRAR_ALGO_ONESHOT: return "k_oneshot";
    case VRAR_ALGO_TWOSTAGE: return "k_twostage";
    case VRAR_ALGO_TWOSTAGE_WRITE: {
      const int wk = write_kernel_for(P, n * elem_size(dtype), g_set.fp8_quant.load() != 0 && dtype != VRAR_FP32);
      return wk == kWriteAsync     ? "k_twostage_write_async"
             : wk == kWriteStaged  ? "k_twostage_write_staged"
             : wk == kWriteBatched ? "k_twostage_write_batched"
                                   : "k_twostage_write";
    }
    case VRAR_ALGO_RD: return wide_wire(algo, dtype) ? "k_rd_wide" : "k_rd";
    case VRAR_ALGO_HIER: return wide_wire(algo, dtype) ? "k_hier_wide" : "k_hier";
    default: return nullptr;
  }
}

int vrar_set_group_size(int L) {
  if (L < 1 || L > kMaxRanks) return VRAR_EINVAL;
  g_set.group_size = L;
  return VRAR_OK;
}
int vrar_get_group_size(void) { return g_set.group_size.load(); }

int vrar_set_rd_chunks(int C) {
  if (C < 1 || C > 8) return VRAR_EINVAL;
  g_set.rd_chunks = C;
  return VRAR_OK;
}
int vrar_get_rd_chunks(void) { return g_set.rd_chunks.load(); }

int vrar_set_edge_sync(int on) {
  g_set.edge_sync = on ? 1 : 0;
  return VRAR_OK;
}
int vrar_get_edge_sync(void) { return g_set.edge_sync.load(); }

int vrar_set_spin_timeout_ns(uint64_t ns) {
  if (ns < 100000ull || ns > 60000000000ull) return VRAR_EINVAL;
  g_set.timeout_ns = ns;
  return VRAR_OK;
}
uint64_t vrar_get_spin_timeout_ns(void) { return g_set.timeout_ns.load(); }

int vrar_query_status(vrar_stream_t stream, uint32_t info[4]) {
  int dev = 0;
  int rc = current_device(&dev);
  if (rc != VRAR_OK) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return cuda_fail(cudaErrorUnknown);
  if (info) std::memset(info, 0, 4 * sizeof(uint32_t));
  uint32_t status = 0;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    Workspace& w = g_ws[dev];
    if (w.ctrl) {
      uint32_t h[kCtrlWords];
      if (cudaMemcpy(h, w.ctrl, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_fail(cudaErrorUnknown);
      if (h[kStatus] != 0) {
        status = h[kStatus];
        if (info) std::memcpy(info, h + kInfo, 4 * sizeof(uint32_t));
        const uint32_t zero[5] = {0, 0, 0, 0, 0};
        if (cudaMemcpy(w.ctrl + kStatus, zero, sizeof(uint32_t), cudaMemcpyHostToDevice) != cudaSuccess ||
            cudaMemcpy(w.ctrl + kInfo, zero, 4 * sizeof(uint32_t), cudaMemcpyHostToDevice) != cudaSuccess)
          return cuda_fail(cudaErrorUnknown);
      }
    }
  }
  // The allocation-free entry point keeps its own control words in its fixed
  // array; a failure there is reported here too (after the workspace's, whose
  // info wins if both failed), and cleared.
  uint32_t h[kCtrlWords];
  bool present = false;
  if ((rc = noalloc_take_status(dev, h, &present)) != VRAR_OK) return rc;
  if (present && h[kStatus] != 0 && status == 0) {
    status = h[kStatus];
    if (info) std::memcpy(info, h + kInfo, 4 * sizeof(uint32_t));
  }
  if (status == 0) return VRAR_OK;
  return status == kErrTimeout ? VRAR_ETIMEDOUT : VRAR_ECUDA;
}

int vrar_reserve(size_t bytes) {
  int dev = 0;
  int rc = current_device(&dev);
  if (rc != VRAR_OK) return rc;
  Workspace* ws = nullptr;
  return ensure_workspace(dev, bytes, &ws);
}

size_t vrar_workspace_bytes(int P, size_t n, vrar_dtype_t dtype, vrar_algo_t algo) {
  if (P < 1 || P > kMaxRanks || !valid_dtype(dtype)) return 0;
  if (algo == VRAR_ALGO_AUTO) algo = static_cast<vrar_algo_t>(select_algo(P, n, dtype));
  const int L = g_set.group_size.load();
  if (check_shape(algo, P, L) != VRAR_OK) return 0;
  if (algo != VRAR_ALGO_RD && algo != VRAR_ALGO_HIER) return 0;
  int dev = 0;
  int sms = 0;
  if (n > 0 && cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices && (sms = device_sms(dev)) > 0) {
    PayloadPlan plan;
    if (plan_payload(algo, P, n, dtype, L, dev, sms, g_set.rd_chunks.load(), false, &plan) == VRAR_OK)
      return plan.bytes;
  }
  cudaGetLastError();
  return 2 * one_round_slot_bytes(algo, P, n, dtype, L);  // no usable device: the bound for any grid
}

int vrar_reset(void) {
  int dev = 0;
  int rc = current_device(&dev);
  if (rc != VRAR_OK) return rc;
  std::lock_guard<std::mutex> lock(g_mu);
  Workspace& w = g_ws[dev];
  if (cudaDeviceSynchronize() != cudaSuccess) return cuda_fail(cudaErrorUnknown);
  if (w.ll) cudaFree(w.ll);
  if (w.ctrl) cudaFree(w.ctrl);
  w = Workspace();
  return VRAR_OK;
}

int vrar_set_max_ctas(int n) {
  if (n < 0) return VRAR_EINVAL;
  g_set.max_ctas = n;
  return VRAR_OK;
}
int vrar_get_max_ctas(void) { return g_set.max_ctas.load(); }

int vrar_set_payload_wire(int wire) {
  if (wire != VRAR_WIRE_ELEMENT && wire != VRAR_WIRE_FP32) return VRAR_EINVAL;
  g_set.payload_wire = wire;
  return VRAR_OK;
}
int vrar_get_payload_wire(void) { return g_set.payload_wire.load(); }

int vrar_set_fp8_quant(int on) {
  g_set.fp8_quant = on ? 1 : 0;
  return VRAR_OK;
}
int vrar_get_fp8_quant(void) { return g_set.fp8_quant.load(); }

int vrar_set_spin_stats(int on) {
  g_set.spin_stats = on ? 1 : 0;
  return VRAR_OK;
}

int vrar_get_spin_stats(uint64_t stats[5], int reset) {
  if (!stats) return VRAR_EINVAL;
  int dev = 0;
  int rc = current_device(&dev);
  if (rc != VRAR_OK) return rc;
  std::memset(stats, 0, 5 * sizeof(uint64_t));
  if (cudaDeviceSynchronize() != cudaSuccess) return cuda_fail(cudaErrorUnknown);
  std::lock_guard<std::mutex> lock(g_mu);
  Workspace& w = g_ws[dev];
  if (!w.ctrl) return VRAR_OK;
  unsigned long long h[kStCount];
  if (cudaMemcpy(h, w.ctrl + kStats, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_fail(cudaErrorUnknown);
  for (int i = 0; i < kStCount; ++i) stats[i] = h[i];
  if (reset && cudaMemset(w.ctrl + kStats, 0, sizeof(h)) != cudaSuccess) return cuda_fail(cudaErrorUnknown);
  return VRAR_OK;
}

int vrar_debug_set_fault_mask(uint32_t mask) {
  g_set.fault_mask = mask;
  return VRAR_OK;
}

const char* vrar_strerror(int code) {
  switch (code) {
    case VRAR_OK: return "success";
    case VRAR_EINVAL: return "invalid argument";
    case VRAR_ENOTSUP: return "shape not supported by the algorithm";
    case VRAR_ENOMEM: return "workspace allocation failed";
    case VRAR_ECUDA: return "CUDA runtime error";
    case VRAR_ETIMEDOUT: return "a device wait timed out";
    case VRAR_ETOOBIG: return "request exceeds the fixed scratch of the allocation-free entry point";
    default: return "unknown error";
  }
}

int vrar_version(void) { return VRAR_VERSION; }

}  // extern "C"

// ---- allocation-free entry point -----------------------------------------------------------
// vrar_allreduce_rd_noalloc runs the k_rd kernel on a fixed array instead of
// the allocated workspace: 256 bytes of control words (ticket, status) and
// then the payload slots. Host code must not pass g_noalloc_scratch itself to
// a kernel (in host code the name is a host-side stand-in, not a device
// address); the device address comes from cudaGetSymbolAddress, looked up
// once per device with that device current.

namespace vrar {
namespace {

constexpr size_t kNoAllocBytes = VRAR_NOALLOC_SCRATCH_BYTES;
constexpr size_t kNoAllocCtrlBytes = 256;
static_assert(kCtrlWords * sizeof(uint32_t) <= kNoAllocCtrlBytes, "control words must fit");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

struct NoAllocDevice {
  unsigned char* base = nullptr;  // device address of g_noalloc_scratch on this device
  int sms = 0;
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc[kMaxDevices];

// Once per device, with that device current: look up the array's device
// address and read the SM count for grid sizing. The array is zero when the
// library's module is loaded; the set-up zeroes it once more on the caller's
// stream (cudaMemsetAsync, ordered before the call's kernel on that stream, so
// it cannot race with it whatever the stream's flags), so that no payload word
// or ticket starts with a value a call could take for its own.
int noalloc_setup(int dev, cudaStream_t stream, NoAllocDevice** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& d = g_noalloc[dev];
  if (!d.base) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e);
    if (cudaMemsetAsync(p, 0, kNoAllocBytes, stream) != cudaSuccess) return cuda_fail(cudaErrorUnknown);
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return cuda_fail(cudaErrorUnknown);
    d.sms = sms;
    d.base = static_cast<unsigned char*>(p);
  }
  *out = &d;
  return VRAR_OK;
}

// The status half of vrar_query_status for the fixed array (declared above).
// The caller has synchronised the stream it asks about.
int noalloc_take_status(int dev, uint32_t* h, bool* present) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  *present = g_noalloc[dev].base != nullptr;
  if (!*present) return VRAR_OK;
  uint32_t* ctrl = reinterpret_cast<uint32_t*>(g_noalloc[dev].base);
  if (cudaMemcpy(h, ctrl, kCtrlWords * sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_fail(cudaErrorUnknown);
  if (h[kStatus] != 0) {
    const uint32_t zero[5] = {0, 0, 0, 0, 0};
    if (cudaMemcpy(ctrl + kStatus, zero, sizeof(uint32_t), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(ctrl + kInfo, zero, 4 * sizeof(uint32_t), cudaMemcpyHostToDevice) != cudaSuccess)
      return cuda_fail(cudaErrorUnknown);
  }
  return VRAR_OK;
}

}  // namespace
}  // namespace vrar

extern "C" int vrar_allreduce_rd_noalloc(const void* const rank_in[], void* const rank_out[], int P, size_t n,
                                         vrar_dtype_t dtype, vrar_stream_t stream) {
  int rc = check_buffers(rank_in, rank_out, P, n, n, dtype);
  if (rc != VRAR_OK) return rc;
  if ((rc = check_shape(VRAR_ALGO_RD, P, 1)) != VRAR_OK) return rc;
  const int64_t items = (static_cast<int64_t>(n) + per_item(dtype) - 1) / per_item(dtype);
  // The documented limit: the one-round slot size must fit beside the control
  // words. The launch planned below never needs more than that.
  if (static_cast<size_t>(items) > kNoAllocBytes ||
      one_round_slot_bytes(VRAR_ALGO_RD, P, n, dtype, 1) > kNoAllocBytes - kNoAllocCtrlBytes)
    return VRAR_ETOOBIG;
  if (n == 0) return VRAR_OK;

  int dev = 0;
  if ((rc = current_device(&dev)) != VRAR_OK) return rc;
  NoAllocDevice* d = nullptr;
  if ((rc = noalloc_setup(dev, reinterpret_cast<cudaStream_t>(stream), &d)) != VRAR_OK) return rc;
  PayloadPlan plan;
  if ((rc = plan_payload(VRAR_ALGO_RD, P, n, dtype, 1, dev, d->sms, g_set.rd_chunks.load(), true, &plan)) != VRAR_OK)
    return rc;
  if (plan.bytes > kNoAllocBytes - kNoAllocCtrlBytes) return VRAR_ETOOBIG;
  KArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int p = 0; p < P; ++p) {
    a.ptr.in[p] = rank_in[p];
    a.ptr.out[p] = rank_out[p];
  }
  a.n = static_cast<int64_t>(n);
  a.items = items;
  a.P = P;
  a.L = 1;
  a.steps = ilog2(P);
  a.chunks = plan.C;
  a.fault_mask = g_set.fault_mask.load();
  a.timeout_ns = g_set.timeout_ns.load();
  a.ctrl = reinterpret_cast<uint32_t*>(d->base);
  a.sig = nullptr;  // recursive doubling uses no barrier rows
  a.ll = reinterpret_cast<uint64_t*>(d->base + kNoAllocCtrlBytes);
  a.slot_items = plan.slot_items;
  a.slot_sets = plan.slot_sets;
  a.B = plan.B;
  return launch(plan.fn, a, a.B * P, reinterpret_cast<cudaStream_t>(stream));
}
