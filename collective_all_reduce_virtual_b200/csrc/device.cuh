// Device-side building blocks of the virtual-rank all-reduce (sm_100a).
//
// Sources (web pages; sections as printed on them):
//  [CAR]   "fix(custom_all_reduce): use SYSTEM scope + ACQUIRE ordering for
//          cross-device signal loads" (ROCm/aiter pull request 4786), "Root
//          cause" and "Changes": per-block start/end signal arrays indexed by
//          [block][rank], written by the peers and polled by the owner; the
//          poll must be an ACQUIRE load at the scope the writers use, and data
//          written with streaming (non-temporal) stores needs a fence before
//          the completion flag.
//  [NVRAR] "Understanding and Improving Communication Performance in
//          Multi-node LLM Inference" (gist.science summary), Methodology item 3:
//          "Fused Payloads" (data and flag in one 8-byte word) and
//          "Sequence-Number Synchronization" (a per-call sequence number
//          instead of a barrier).
//
// All virtual ranks live on one device, so every flag and payload access is
// at .gpu scope: the same-device counterpart of the SYSTEM scope that [CAR]
// needs across devices.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace vrar {

constexpr int kMaxRanks = 32;
#ifndef VRAR_THREADS
#define VRAR_THREADS 512
#endif
constexpr int kThreads = VRAR_THREADS;  // threads per CTA of every kernel
constexpr int kMaxCtas = 2048;         // grid cap; sizes the signal arrays
constexpr int kSigPhaseWords = kMaxCtas * kMaxRanks;
constexpr int kPhases = 3;             // start, mid, end

// Control words at the start of the workspace (32-bit words).
enum Ctrl : int {
  kTicket = 0,     // 64-bit ticket (words 0-1): high half = calls completed, low half = CTAs arrived
  kStatus = 2,     // sticky error code (0 = none) until the host reads it
  kFailEpoch = 3,  // sequence number of a call in which some wait gave up
  kInfo = 4,       // 4 words: failing call, phase, rank, block
  kStats = 16,     // 5 x 64-bit spin statistics (see record_spins), words 16..25
  kCtrlWords = 32
};

// Spin statistics counters (64-bit, at ctrl + kStats).
enum StatIdx : int { kStWaits = 0, kStSpins = 1, kStMax = 2, kStLong = 3, kStTimeouts = 4, kStCount = 5 };
constexpr uint32_t kLongWaitSpins = 16384;

enum Phase : uint32_t { kPhStart = 1, kPhMid = 2, kPhEnd = 3, kPhPayload = 4, kPhCopy = 5 };
constexpr uint32_t kErrTimeout = 1;

struct RankPtrs {
  const void* in[kMaxRanks];
  void* out[kMaxRanks];
};

// Kernel arguments, passed by value (they live in the constant bank).
struct KArgs {
  RankPtrs ptr;
  int64_t n;         // elements per rank (the full vector)
  int64_t items;     // 16-byte items per rank: ceil(n / elements-per-item)
  int P;             // virtual ranks
  int B;             // CTAs per rank
  int L;             // group size (hierarchical)
  int steps;         // recursive-doubling steps (log2 of the ranks doubled over)
  int chunks;        // payload pieces in flight per thread and step
  int edge_sync;     // run start/end barriers
  int stages;        // shared-memory pipeline depth (staged kernels)
  uint32_t fault_mask;
  uint64_t timeout_ns;
  uint32_t* ctrl;
  uint32_t* sig;     // kPhases x kSigPhaseWords flag words
  uint64_t* ll;      // payload slots
  int64_t slot_items;  // payload slots (32 bytes each) per rank, step and slot set
  int slot_sets;       // 1: slot = item index (one round); 2: slots reused by round parity
  int prefetch_next;   // hierarchical: warm L2 with the next round's inputs
  unsigned long long* stats;  // spin statistics, or null when they are off
};

// ---- PTX wrappers --------------------------------------------------------------

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Inputs: read-only for the whole launch, read once per CTA -> non-coherent
// path without L1 allocation.
__device__ __forceinline__ uint4 ld_input(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// The same load, kept in program order with the other volatile accesses: a
// batch of these is issued as written, before the arithmetic that uses it.
__device__ __forceinline__ uint4 ld_input_ordered(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Data another CTA of this launch wrote (read after an acquire): L2 only.
__device__ __forceinline__ uint4 ld_peer(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ void st_plain(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Streaming store (evict-first), the CUDA counterpart of a non-temporal store.
__device__ __forceinline__ void st_stream(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Four fused payload words (one 32-byte slot, 32-byte aligned) in one 256-bit
// access, which sm_100 has for global memory. A vector access is performed as
// accesses of its 8-byte elements, each single-copy atomic, in no fixed order:
// the reader still checks the tag of every word.
__device__ __forceinline__ void st_payload4(uint64_t* p, uint64_t a, uint64_t b, uint64_t c, uint64_t d) {
  asm volatile("st.relaxed.gpu.global.v4.u64 [%0], {%1,%2,%3,%4};" ::"l"(p), "l"(a), "l"(b), "l"(c), "l"(d)
               : "memory");
}

__device__ __forceinline__ void ld_payload4(const uint64_t* p, uint64_t& a, uint64_t& b, uint64_t& c, uint64_t& d) {
  asm volatile("ld.relaxed.gpu.global.v4.u64 {%0,%1,%2,%3}, [%4];" : "=l"(a), "=l"(b), "=l"(c), "=l"(d) : "l"(p)
               : "memory");
}

// ---- shared-memory pipelines: mbarriers and bulk copies (no multicast) -------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async proxy (the bulk copies).
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// One bulk copy global -> this CTA's shared memory, completing `bytes` of the
// barrier's transaction count. 16-byte aligned addresses, bytes % 16 == 0.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Per-thread asynchronous 16-byte copy global -> shared (L2 only), and its
// group bookkeeping: commit the copies issued so far as one group; wait until
// at most N groups of this thread are still in flight.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(smem_u32(p)));
  return v;
}

// ---- element types ----------------------------------------------------------------
// An "item" is 16 bytes of one rank's vector: 8 bf16 or 4 fp32 elements.

struct Bf16T {
  using E = uint16_t;
  static constexpr int VE = 8;
  __device__ __forceinline__ static void widen(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ __forceinline__ static uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static uint4 narrow(const float (&f)[8]) {
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
  }
  __device__ __forceinline__ static float elem_to_f(E e) { return __uint_as_float(static_cast<uint32_t>(e) << 16); }
  __device__ __forceinline__ static E f_to_elem(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<E*>(&h);
  }
};

// IEEE binary16: widening is exact (cvt.f32.f16), narrowing is round to
// nearest even with subnormals kept (cvt.rn.f16x2.f32).
struct F16T {
  using E = uint16_t;
  static constexpr int VE = 8;
  __device__ __forceinline__ static void widen(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
      f[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
    }
  }
  __device__ __forceinline__ static uint32_t pack2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ __forceinline__ static uint4 narrow(const float (&f)[8]) {
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
  }
  __device__ __forceinline__ static float elem_to_f(E e) { return __half2float(__ushort_as_half(e)); }
  __device__ __forceinline__ static E f_to_elem(float f) { return __half_as_ushort(__float2half_rn(f)); }
};

struct F32T {
  using E = float;
  static constexpr int VE = 4;
  __device__ __forceinline__ static void widen(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 narrow(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
  __device__ __forceinline__ static float elem_to_f(E e) { return e; }
  __device__ __forceinline__ static E f_to_elem(float f) { return f; }
};

// ---- fp8 payloads (a reading of the custom all-reduce's ca_fp8_quant flag) ----------------
// Every value that passes from one rank to another travels as OCP FP8 E4M3
// with one binary32 scale per group of 8 elements, which is one 16-byte item
// of a 16-bit tensor: s = amax / 448 (amax the group's largest magnitude; 1 if
// the division gives 0), q = E4M3(x / s) rounded to nearest even and saturated
// at 448, and the receiver's value is q * s. On one device the values never
// need to be stored in fp8: each kernel quantises and dequantises in
// registers where the value would cross between ranks, and moves the same
// bytes as without fp8.

// E4M3 rounding of two binary32 values and back: cvt.rn.satfinite.e4m3x2.f32
// packs (hi, lo) into two bytes; cvt.rn.f16x2.e4m3x2 widens them exactly to
// two halves (every E4M3 value is a binary16 value), which widen exactly to
// binary32.
__device__ __forceinline__ void e4m3_round2(float& lo, float& hi) {
  uint16_t q;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(q) : "f"(hi), "f"(lo));
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(q));
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

// The group scale amax / 448, rounded to nearest even, for 2^-120 <= amax <=
// FLT_MAX: the product by c = RN(1/448) = 0x1.24924ap-9, corrected once by its
// exact remainder (Markstein's FMA correction step: r = x - q0 * 448 is exact
// in one fma, and q0 + r * c rounds to the quotient). Checked against the
// exactly rounded quotient for every binary32 in that range (the test suite
// runs the same formula over all of them); below 2^-120 the quotient is deep in
// the subnormal range, where the correction can be off by one unit, and the
// caller divides instead.
__device__ __forceinline__ float div448_rn(float x) {
  const float c = 0x1.24924ap-9f;
  const float q0 = __fmul_rn(x, c);
  const float r = __fmaf_rn(-q0, 448.0f, x);
  return __fmaf_rn(r, c, q0);
}

// 1/s to within 2^-23 relative, for s and 1/s normal: the hardware's
// approximate reciprocal and one Newton-Raphson step (e = 1 - s r0 in one fma,
// r1 = r0 + r0 e), whose error is the square of the approximation's plus one
// rounding.
__device__ __forceinline__ float recip_nr(float s) {
  float r0;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r0) : "f"(s));
  const float e = __fmaf_rn(-s, r0, 1.0f);
  return __fmaf_rn(r0, e, r0);
}

// E4M3(x / s) needs the binary32 quotient x / s only up to which side of an
// E4M3 rounding midpoint it falls. The product t = x * r with r within 2^-23
// of 1/s (relative) is within 3 units in the last place of the quotient (that
// error and one rounding of 2^-24), so it rounds to the same E4M3 value
// unless a midpoint lies within 3 units of it. Where t
// is within 8 units of a midpoint of a normal E4M3 binade (its 20 fraction bits
// below the 3 that E4M3 keeps are within 8 of 1000...0), or in E4M3's
// subnormal range (below 2^-6, where the midpoints sit elsewhere), the exact
// quotient is taken instead. Binade edges are E4M3 values, not midpoints, so
// a t on the other side of one from the quotient still rounds the same way.
__device__ __forceinline__ float fp8_quotient(float x, float s, float r) {
  const float t = __fmul_rn(x, r);
  const uint32_t u = __float_as_uint(t) & 0x7FFFFFFFu;
  const int32_t below = static_cast<int32_t>(u & 0xFFFFFu) - 0x80000;
  if ((u != 0u && u < 0x3C800000u) || (below >= -8 && below <= 8)) return __fdiv_rn(x, s);
  return t;
}

// The fp8 wire on one group of 8 binary32 values, in place: s = amax / 448
// (1 when that is 0), each value quantised to E4M3(x / s) and received as
// E4M3 * s, with binary32 division and product rounded to nearest even
// (the scale as div448_rn gives it, __fmul_rn; the quotient as fp8_quotient
// gives it). Scales outside [2^-125, 2^125] (whose reciprocal is not a normal
// number) divide every value exactly.
__device__ __forceinline__ void fp8_qdq8(float (&f)[8]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
  float s = (amax >= 0x1p-120f && amax <= 0x1.fffffep127f) ? div448_rn(amax) : __fdiv_rn(amax, 448.0f);
  if (s == 0.0f) s = 1.0f;
  const bool fast = s >= 0x1p-125f && s <= 0x1p125f;
  const float r = fast ? recip_nr(s) : 0.0f;
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    float lo = fast ? fp8_quotient(f[i], s, r) : __fdiv_rn(f[i], s);
    float hi = fast ? fp8_quotient(f[i + 1], s, r) : __fdiv_rn(f[i + 1], s);
    e4m3_round2(lo, hi);
    f[i] = __fmul_rn(lo, s);
    f[i + 1] = __fmul_rn(hi, s);
  }
}

// fp32 accumulator of one item. Every add is add.rn.f32: round to nearest
// even, never contracted into an FMA, subnormals kept (no .ftz).
// init_in / add_in take an input item as it arrives from a rank (through the
// fp8 wire when kQ8); round_out rounds the sum for an all-gather that crosses
// ranks (through the fp8 wire again when kQ8).
template <class D>
struct Acc {
  float v[D::VE];
  __device__ __forceinline__ void init(const uint4& x) { D::widen(x, v); }
  __device__ __forceinline__ void add(const uint4& x) {
    float f[D::VE];
    D::widen(x, f);
#pragma unroll
    for (int i = 0; i < D::VE; ++i) v[i] = __fadd_rn(v[i], f[i]);
  }
  __device__ __forceinline__ uint4 round() const { return D::narrow(v); }

  template <bool kQ8>
  __device__ __forceinline__ void init_in(const uint4& x) {
    D::widen(x, v);
    if constexpr (kQ8) fp8_qdq8(v);
  }
  template <bool kQ8>
  __device__ __forceinline__ void add_in(const uint4& x) {
    float f[D::VE];
    D::widen(x, f);
    if constexpr (kQ8) fp8_qdq8(f);
#pragma unroll
    for (int i = 0; i < D::VE; ++i) v[i] = __fadd_rn(v[i], f[i]);
  }
  template <bool kQ8>
  __device__ __forceinline__ uint4 round_out() const {
    if constexpr (kQ8) {
      float t[D::VE];
#pragma unroll
      for (int i = 0; i < D::VE; ++i) t[i] = v[i];
      fp8_qdq8(t);
      return D::narrow(t);
    } else {
      return D::narrow(v);
    }
  }
};

// rnd(f(a) + f(b)) element-wise: one recursive-doubling combine.
template <class D>
__device__ __forceinline__ uint4 add_round(const uint4& a, const uint4& b) {
  Acc<D> acc;
  acc.init(a);
  acc.add(b);
  return acc.round();
}

// ---- item I/O with a ragged tail ----------------------------------------------------
// Item `it` of a rank vector of n elements; the last item may hold fewer than
// VE elements. Missing elements load as zero and are never stored.

template <class D>
__device__ __forceinline__ int item_valid(int64_t it, int64_t n) {
  const int64_t rem = n - it * D::VE;
  return rem >= D::VE ? D::VE : static_cast<int>(rem);
}

template <class D>
__device__ __forceinline__ uint4 load_item_input(const void* base, int64_t it, int64_t n) {
  const typename D::E* p = static_cast<const typename D::E*>(base) + it * D::VE;
  const int nv = item_valid<D>(it, n);
  if (nv == D::VE) return ld_input(p);
  union { uint4 u; typename D::E e[D::VE]; } t;
#pragma unroll
  for (int i = 0; i < D::VE; ++i) t.e[i] = i < nv ? p[i] : typename D::E(0);
  return t.u;
}

template <class D>
__device__ __forceinline__ uint4 load_item_peer(const void* base, int64_t it, int64_t n) {
  const typename D::E* p = static_cast<const typename D::E*>(base) + it * D::VE;
  const int nv = item_valid<D>(it, n);
  if (nv == D::VE) return ld_peer(p);
  union { uint4 u; typename D::E e[D::VE]; } t;
#pragma unroll
  for (int i = 0; i < D::VE; ++i) t.e[i] = i < nv ? static_cast<const volatile typename D::E*>(p)[i] : typename D::E(0);
  return t.u;
}

template <class D, bool kStream>
__device__ __forceinline__ void store_item(void* base, int64_t it, int64_t n, const uint4& v) {
  typename D::E* p = static_cast<typename D::E*>(base) + it * D::VE;
  const int nv = item_valid<D>(it, n);
  if (nv == D::VE) {
    if (kStream) st_stream(p, v); else st_plain(p, v);
    return;
  }
  union { uint4 u; typename D::E e[D::VE]; } t;
  t.u = v;
#pragma unroll
  for (int i = 0; i < D::VE; ++i)
    if (i < nv) p[i] = t.e[i];
}

// Item `it` stored to `count` outputs rank_out[first + (start + j) mod count]
// for j = 0 .. count-1 (streaming stores): the full-item check is made once.
template <class D>
__device__ __forceinline__ void store_item_rotated(void* const* out, int first, int count, int start, int64_t it,
                                                   int64_t n, const uint4& v) {
  if ((it + 1) * D::VE <= n) {
    int q = start;
    for (int j = 0; j < count; ++j) {
      st_stream(static_cast<typename D::E*>(out[first + q]) + it * D::VE, v);
      q = q + 1 == count ? 0 : q + 1;
    }
    return;
  }
  for (int j = 0; j < count; ++j) {
    const int q = start + j >= count ? start + j - count : start + j;
    store_item<D, true>(out[first + q], it, n, v);
  }
}

// Ascending-rank fp32 sum of item `it` over ranks first .. first+count-1 (not
// rounded), each input through the fp8 wire when kQ8. Loads are issued eight
// at a time so that they overlap; the adds stay in rank order.
template <class D, bool kQ8 = false>
__device__ __forceinline__ Acc<D> reduce_item_acc(const RankPtrs& rp, int first, int count, int64_t it, int64_t n) {
  Acc<D> acc;
  for (int q0 = 0; q0 < count; q0 += 8) {
    uint4 x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (q0 + j < count) x[j] = load_item_input<D>(rp.in[first + q0 + j], it, n);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (q0 + j < count) {
        if (q0 + j == 0) acc.template init_in<kQ8>(x[j]); else acc.template add_in<kQ8>(x[j]);
      }
    }
  }
  return acc;
}

// The same sum rounded once to the element type.
template <class D, bool kQ8 = false>
__device__ __forceinline__ uint4 reduce_item(const RankPtrs& rp, int first, int count, int64_t it, int64_t n) {
  return reduce_item_acc<D, kQ8>(rp, first, count, it, n).round();
}

// The sum as the 2-stage kernels hand it to the other ranks: through the fp8
// wire a second time when kQ8, then rounded to the element type.
template <class D, bool kQ8>
__device__ __forceinline__ uint4 reduce_item_out(const RankPtrs& rp, int first, int count, int64_t it, int64_t n) {
  return reduce_item_acc<D, kQ8>(rp, first, count, it, n).template round_out<kQ8>();
}

// A 16-byte item of a 16-bit type as fp32 partials: two quads of 4 floats.
__device__ __forceinline__ void floats_to_quads(const float (&f)[8], uint4& q0, uint4& q1) {
  q0 = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  q1 = make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]), __float_as_uint(f[6]), __float_as_uint(f[7]));
}

template <class D>
__device__ __forceinline__ uint4 quads_to_item(const uint4& q0, const uint4& q1) {
  const float f[8] = {__uint_as_float(q0.x), __uint_as_float(q0.y), __uint_as_float(q0.z), __uint_as_float(q0.w),
                      __uint_as_float(q1.x), __uint_as_float(q1.y), __uint_as_float(q1.z), __uint_as_float(q1.w)};
  return D::narrow(f);
}

// ---- launch ordering -------------------------------------------------------------------
// Kernels are launched with programmatic stream serialisation: the next call's
// grid may be scheduled while this one drains, and it waits in
// griddepcontrol.wait until this grid has completed and its memory is visible.
// Every kernel executes pdl_wait() before its first global memory access.
// A grid's dependents launch only once all its CTAs have triggered, i.e. once
// they are all resident, so the co-residency the waits below rely on holds.

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// L2 prefetch hint for [p, p + bytes) (16-byte aligned, bytes a multiple of 16).
// Kernels issue these for their first inputs between pdl_trigger() and
// pdl_wait(), i.e. while the previous call may still be running: a prefetch
// returns no data to the thread, and L2 is the point of coherence of the
// device, so a line fetched early is updated by any later write to it and no
// thread can see a stale value. It only moves DRAM latency off the critical
// path of back-to-back calls.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Prefetch items [first, first + count) of a rank vector of n elements,
// clipped to the items that lie wholly inside the vector.
template <class D>
__device__ __forceinline__ void prefetch_items(const void* base, int64_t first, int64_t count, int64_t n) {
  const int64_t full = n / D::VE;
  const int64_t last = first + count < full ? first + count : full;
  if (last > first)
    prefetch_l2(static_cast<const char*>(base) + first * 16, static_cast<uint32_t>((last - first) * 16));
}

// ---- per-call sequence number [NVRAR "Sequence-Number Synchronization"] ------------------
// One 64-bit ticket per device: every CTA of a call adds 1 (a relaxed atomic:
// the ticket is the only location involved, and its modification order
// serialises the adds). The CTA that sees the low half reach gridDim.x - 1 is
// the last to arrive, and adds 2^32 - gridDim.x: the call count goes up by one
// and the arrival count back to 0, for the next launch (stream order). Every
// CTA of a call therefore reads the same call count c and uses
// (c mod (2^31 - 1)) + 1 as the call's flag: never 0 (the value of a
// never-written word) and below 2^31, so that payload tags can carry a lap bit
// in bit 31 (see rd_tag). Flags grow by one per call that uses them, so a flag
// or payload word left by any earlier call never equals the current flag
// (until 2^31 - 1 calls wrap it). Kernels that use no flags never touch the
// ticket.

struct Cta {
  int r;          // virtual rank this CTA acts for
  int b;          // index of the CTA within its rank
  uint32_t flag;  // this call's sequence number (never 0)
};

__device__ __forceinline__ Cta cta_coords(const KArgs& a) {
  Cta c;
  c.r = static_cast<int>(blockIdx.x % a.P);
  c.b = static_cast<int>(blockIdx.x / a.P);
  c.flag = 0;
  return c;
}

// Thread 0 takes the ticket (issue this early: the result is needed only by
// cta_publish_flag, so the atomic's latency overlaps the first data loads).
__device__ __forceinline__ unsigned long long cta_take_ticket(const KArgs& a) {
  unsigned long long old = 0;
  if (threadIdx.x == 0) {
    unsigned long long* t = reinterpret_cast<unsigned long long*>(a.ctrl + kTicket);
    old = atomicAdd(t, 1ull);
    if (static_cast<uint32_t>(old) == gridDim.x - 1) atomicAdd(t, (1ull << 32) - gridDim.x);
  }
  return old;
}

// Broadcast the call's flag to the whole CTA (contains a CTA barrier).
__device__ __forceinline__ void cta_publish_flag(Cta& c, unsigned long long ticket) {
  __shared__ uint32_t s_flag;
  if (threadIdx.x == 0) s_flag = static_cast<uint32_t>(ticket >> 32) % 0x7FFFFFFFu + 1u;
  __syncthreads();
  c.flag = s_flag;
}

// Spin statistics of the cross-rank waits, after the temporary instrumentation
// described in [CAR] "Validation": per wait, the number of polls it took; the
// counters keep the number of waits, the total and largest poll count, the
// waits of kLongWaitSpins polls or more, and the waits that hit the time limit
// (the "safety net"). Off unless the host turned it on (a.stats non-null).
// The threads of a warp that finish a wait together are combined first, so a
// warp costs one set of atomics, not 32.
__device__ __forceinline__ void record_spins(const KArgs& a, uint32_t spins, bool timed_out) {
  if (!a.stats) return;
  const unsigned m = __activemask();
  const uint32_t sum = __reduce_add_sync(m, spins);
  const uint32_t mx = __reduce_max_sync(m, spins);
  const uint32_t nlong = __reduce_add_sync(m, spins >= kLongWaitSpins ? 1u : 0u);
  const uint32_t nto = __reduce_add_sync(m, timed_out ? 1u : 0u);
  if ((threadIdx.x & 31) == static_cast<unsigned>(__ffs(m) - 1)) {
    atomicAdd(a.stats + kStWaits, static_cast<unsigned long long>(__popc(m)));
    atomicAdd(a.stats + kStSpins, static_cast<unsigned long long>(sum));
    atomicMax(a.stats + kStMax, static_cast<unsigned long long>(mx));
    if (nlong) atomicAdd(a.stats + kStLong, static_cast<unsigned long long>(nlong));
    if (nto) atomicAdd(a.stats + kStTimeouts, static_cast<unsigned long long>(nto));
  }
}

__device__ __forceinline__ void report_timeout(const KArgs& a, const Cta& c, uint32_t phase) {
  if (atomicCAS(a.ctrl + kStatus, 0u, kErrTimeout) == 0u) {
    a.ctrl[kInfo + 0] = c.flag;
    a.ctrl[kInfo + 1] = phase;
    a.ctrl[kInfo + 2] = static_cast<uint32_t>(c.r);
    a.ctrl[kInfo + 3] = static_cast<uint32_t>(c.b);
  }
  st_relaxed(a.ctrl + kFailEpoch, c.flag);
}

// Poll `p` with acquire loads until it equals this call's flag. Gives up when
// the time limit passes or another CTA of this call has given up; returns
// false then. Equality (not >=) keeps the test valid across 32-bit wrap.
__device__ __forceinline__ bool wait_flag(const uint32_t* p, const KArgs& a, const Cta& c, uint32_t phase) {
  uint32_t polls = 1;
  bool ok = true;
  if (ld_acquire(p) != c.flag) {
    const uint64_t t0 = globaltimer_ns();
    for (;; ++polls) {
      if (ld_acquire(p) == c.flag) break;
      if ((polls & 63u) == 0u) {
        if (ld_relaxed(a.ctrl + kFailEpoch) == c.flag) {
          ok = false;
          break;
        }
        if (globaltimer_ns() - t0 > a.timeout_ns) {
          report_timeout(a, c, phase);
          record_spins(a, polls, true);
          return false;
        }
      }
    }
  }
  record_spins(a, polls, false);
  return ok;
}

// Block barrier across ranks [CAR start_sync / end_sync]: block b of rank r
// posts the call's flag into slot [r] of block b's signal row of every rank p,
// then polls its own row until all P entries carry the flag. Threads 0..P-1
// do one rank each. The CTA barrier before the post orders all of the CTA's
// earlier stores before the release; the one after the poll extends the
// acquire to the whole CTA. Returns false if any wait gave up.
__device__ __forceinline__ bool block_barrier(const KArgs& a, const Cta& c, uint32_t phase) {
  __syncthreads();
  bool fail = false;
  if (threadIdx.x < a.P) {
    const int p = threadIdx.x;
    uint32_t* sig = a.sig + static_cast<size_t>(phase - 1) * kSigPhaseWords;
    if (!((a.fault_mask >> c.r) & 1u))
      st_release(sig + (static_cast<size_t>(p) * a.B + c.b) * kMaxRanks + c.r, c.flag);
    fail = !wait_flag(sig + (static_cast<size_t>(c.r) * a.B + c.b) * kMaxRanks + p, a, c, phase);
  }
  return __syncthreads_or(fail) == 0;
}

// ---- fused payload words [NVRAR "Fused Payloads"] ---------------------------------------
// One item (16 data bytes) travels as four 8-byte words {low: 4 data bytes,
// high: the call's sequence number}; a word is valid once its high half equals
// the flag, so no separate signal is needed.

__device__ __forceinline__ void send_item(uint64_t* slot, const uint4& v, uint32_t flag) {
  const uint64_t hi = static_cast<uint64_t>(flag) << 32;
  st_payload4(slot, hi | v.x, hi | v.y, hi | v.z, hi | v.w);
}

}  // namespace vrar
