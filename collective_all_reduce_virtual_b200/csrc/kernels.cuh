// The all-reduce kernels. One launch does the work of all P virtual ranks:
// CTA blockIdx.x acts as block b = blockIdx.x / P of rank r = blockIdx.x % P,
// every rank has the same number B of CTAs, and the grid is sized so that all
// CTAs are resident at once (the waits below need every peer to be running).
//
// Work split: within a rank, thread t of block b takes the items
// b*T + t, b*T + t + B*T, ... of whatever range the phase covers (T =
// kThreads). Every rank uses the same split, so a CTA only ever waits on the
// CTAs with its own block index b in the other ranks.
//
// Sources: see device.cuh ([CAR] pull request 4786 for the custom all-reduce
// one-shot / 2-stage / write mode and its start/end barriers; [NVRAR]
// Methodology item 3 for the three-phase hierarchical algorithm, recursive
// doubling, chunking, fused payloads and sequence numbers).
#pragma once

#include "device.cuh"

namespace vrar {

__device__ __forceinline__ int64_t lo_of(int64_t part, int64_t piece, int64_t total) {
  const int64_t v = part * piece;
  return v < total ? v : total;
}

// (a + b) mod m for 0 <= a, b < m, without an integer division: the rotated
// rank orders below (stores and peer reads staggered by the rank's own index,
// so that the ranks do not all touch one buffer at once) are computed per item.
__device__ __forceinline__ int add_mod(int a, int b, int m) {
  const int v = a + b;
  return v >= m ? v - m : v;
}

// One-shot [CAR, the 1-stage kernel]: every rank reads all P inputs and
// reduces the whole vector into its own output, between start and end
// barriers. The P CTAs with the same b read the same items at about the same
// time, so all but the first read of each line hit L2. T threads per CTA:
// small messages run faster as more, smaller CTAs. kQ8: every input passes
// the fp8 wire once (every rank reads all P inputs through it).
template <class D, int T = kThreads, bool kQ8 = false>
__global__ void __launch_bounds__(T, 2) k_oneshot(const KArgs a) {
  pdl_trigger();
  Cta c = cta_coords(a);
  // Rank r's CTAs prefetch input r only: all P ranks read the same items.
  if (threadIdx.x == 0)
    prefetch_items<D>(a.ptr.in[c.r], static_cast<int64_t>(c.b) * T, T, a.n);
  pdl_wait();
  if (a.edge_sync) {
    cta_publish_flag(c, cta_take_ticket(a));
    if (!block_barrier(a, c, kPhStart)) return;
  }
  const int64_t stride = static_cast<int64_t>(a.B) * T;
  void* out = a.ptr.out[c.r];
  for (int64_t it = static_cast<int64_t>(c.b) * T + threadIdx.x; it < a.items; it += stride)
    store_item<D, true>(out, it, a.n, reduce_item<D, kQ8>(a.ptr, 0, a.P, it, a.n));
  if (a.edge_sync) block_barrier(a, c, kPhEnd);
}

// 2-stage [CAR "cross_device_reduce_2stage"], pull mode. Stage 1: rank r
// reduces slice r (ceil(items / P) items) over all P inputs into out[r]. Mid
// barrier. Stage 2: rank r copies every other slice s out of out[s]. T threads
// per CTA (the library launches 256: more, smaller CTAs per column barrier).
// kQ8: the inputs pass the fp8 wire for stage 1 and the reduced slice passes
// it again for stage 2; the owner stores that value too.
template <class D, int T = kThreads, bool kQ8 = false>
__global__ void __launch_bounds__(T) k_twostage(const KArgs a) {
  pdl_trigger();
  Cta c = cta_coords(a);
  {
    const int64_t piece = (a.items + a.P - 1) / a.P;
    const int64_t first = lo_of(c.r, piece, a.items) + static_cast<int64_t>(c.b) * T;
    const int64_t count = min(static_cast<int64_t>(T), lo_of(c.r + 1, piece, a.items) - first);
    if (threadIdx.x < a.P) prefetch_items<D>(a.ptr.in[threadIdx.x], first, count, a.n);
  }
  pdl_wait();
  const unsigned long long ticket = cta_take_ticket(a);
  if (a.edge_sync) {
    cta_publish_flag(c, ticket);
    if (!block_barrier(a, c, kPhStart)) return;
  }
  const int64_t stride = static_cast<int64_t>(a.B) * T;
  const int64_t t0 = static_cast<int64_t>(c.b) * T + threadIdx.x;
  const int64_t piece = (a.items + a.P - 1) / a.P;
  void* own = a.ptr.out[c.r];
  {
    const int64_t lo = lo_of(c.r, piece, a.items), hi = lo_of(c.r + 1, piece, a.items);
    for (int64_t it = lo + t0; it < hi; it += stride)
      store_item<D, false>(own, it, a.n, reduce_item_out<D, kQ8>(a.ptr, 0, a.P, it, a.n));
  }
  if (!a.edge_sync) cta_publish_flag(c, ticket);
  if (!block_barrier(a, c, kPhMid)) return;
  for (int64_t off = t0; off < piece; off += stride) {
    // Up to 8 peer slices per batch so that the loads overlap; sources are
    // staggered (r+1, r+2, ...) so the ranks do not all read one slice at once.
    for (int j0 = 1; j0 < a.P; j0 += 8) {
      uint4 v[8];
      int64_t it[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int s = add_mod(c.r, j0 + j < a.P ? j0 + j : 0, a.P);  // lanes past P are skipped below
        it[j] = s * piece + off;
        if (j0 + j < a.P && it[j] < lo_of(s + 1, piece, a.items)) v[j] = load_item_peer<D>(a.ptr.out[s], it[j], a.n);
        else it[j] = -1;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j0 + j < a.P && it[j] >= 0) store_item<D, true>(own, it[j], a.n, v[j]);
    }
  }
  if (a.edge_sync) block_barrier(a, c, kPhEnd);
}

// 2-stage write mode [CAR "cross_device_reduce_2stage_write_mode", Root cause
// and change 3]: rank r reduces slice r and streams the result straight into
// all P outputs; a device-scope fence then makes those stores visible before
// the end barrier's flags. kQ8: inputs and reduced slice pass the fp8 wire.
template <class D, bool kQ8>
__device__ __forceinline__ void twostage_write_plain(const KArgs& a) {
  pdl_trigger();
  Cta c = cta_coords(a);
  {
    const int64_t piece = (a.items + a.P - 1) / a.P;
    const int64_t first = lo_of(c.r, piece, a.items) + static_cast<int64_t>(c.b) * kThreads;
    const int64_t count = min(static_cast<int64_t>(kThreads), lo_of(c.r + 1, piece, a.items) - first);
    if (threadIdx.x < a.P) prefetch_items<D>(a.ptr.in[threadIdx.x], first, count, a.n);
  }
  pdl_wait();
  if (a.edge_sync) {
    cta_publish_flag(c, cta_take_ticket(a));
    if (!block_barrier(a, c, kPhStart)) return;
  }
  const int64_t stride = static_cast<int64_t>(a.B) * kThreads;
  const int64_t piece = (a.items + a.P - 1) / a.P;
  const int64_t lo = lo_of(c.r, piece, a.items), hi = lo_of(c.r + 1, piece, a.items);
  for (int64_t it = lo + static_cast<int64_t>(c.b) * kThreads + threadIdx.x; it < hi; it += stride) {
    store_item_rotated<D>(a.ptr.out, 0, a.P, c.r, it, a.n, reduce_item_out<D, kQ8>(a.ptr, 0, a.P, it, a.n));
  }
  if (a.edge_sync) {
    __threadfence();
    block_barrier(a, c, kPhEnd);
  }
}

// The plain write kernel, registers left to the compiler (78 for bf16): one
// 512-thread CTA per SM, the build that streams DRAM-sized calls best.
template <class D, bool kQ8 = false>
__global__ void __launch_bounds__(kThreads) k_twostage_write(const KArgs a) {
  twostage_write_plain<D, kQ8>(a);
}

// The same kernel with its registers budgeted for kMinBlocks CTAs per SM, for
// small calls that one CTA per SM cannot cover in one pass (same name: an
// overload of the template above by its parameter list).
template <class D, bool kQ8, int kMinBlocks>
__global__ void __launch_bounds__(kThreads, kMinBlocks) k_twostage_write(const KArgs a) {
  twostage_write_plain<D, kQ8>(a);
}

// 2-stage write mode for large messages, with IT items per thread in flight.
// Same result and work split by rank as k_twostage_write: CTA b of rank r
// takes passes b, b+B, ... of slice r, a pass being kBatchThreads * IT items
// (warp w covers items w*32*IT ... of the pass, lane l items l, l+32, ...).
// For each pass a thread issues the loads of its IT items from eight input
// ranks at a time before the first add of that batch, so each thread keeps
// 8 * IT * 16 bytes in flight without shared memory or synchronisation, and
// the stores of one pass overlap the loads of the next. Rank indices are
// compile-time (kMaxP is 8, 16 or 32, ranks past P skipped), so the rank
// pointers are read straight from the kernel parameters. Every full pass runs
// the unguarded loop; at most one pass per CTA (the one that reaches the end
// of the slice or the ragged last item) takes the per-item path.
// Threads per CTA and the CTAs per SM its register budget is sized for
// (compile-time; the defaults, two 256-thread CTAs per SM, measured fastest).
#ifndef VRAR_BATCH_THREADS
#define VRAR_BATCH_THREADS 256
#endif
#ifndef VRAR_BATCH_MINB
#define VRAR_BATCH_MINB 2
#endif
constexpr int kBatchThreads = VRAR_BATCH_THREADS;

template <class D, int IT, int kMaxP, bool kQ8 = false>
__global__ void __launch_bounds__(kBatchThreads, VRAR_BATCH_MINB) k_twostage_write_batched(const KArgs a) {
  constexpr int kSpan = kBatchThreads * IT;
  pdl_trigger();
  Cta c = cta_coords(a);
  const int64_t piece = (a.items + a.P - 1) / a.P;
  const int64_t lo = lo_of(c.r, piece, a.items), hi = lo_of(c.r + 1, piece, a.items);
  const int64_t first = lo + static_cast<int64_t>(c.b) * kSpan;
  if (threadIdx.x < a.P && first < hi)
    prefetch_items<D>(a.ptr.in[threadIdx.x], first, min(static_cast<int64_t>(kSpan), hi - first), a.n);
  pdl_wait();
  if (a.edge_sync) {
    cta_publish_flag(c, cta_take_ticket(a));
    if (!block_barrier(a, c, kPhStart)) return;
  }
  const int64_t full_hi = min(hi, a.n / D::VE);  // items of the slice wholly inside the vector
  const int64_t stride = static_cast<int64_t>(a.B) * kSpan;
  const int64_t lane_off = (threadIdx.x >> 5) * 32 * IT + (threadIdx.x & 31);
  int64_t base = first;
  for (; base + kSpan <= full_hi; base += stride) {
    const int64_t i0 = base + lane_off;  // this thread's items: i0 + 32 t, t < IT
    Acc<D> acc[IT];
#pragma unroll
    for (int q0 = 0; q0 < kMaxP; q0 += 8) {
      if (q0 < a.P) {
        uint4 x[IT][8];
#pragma unroll
        for (int t = 0; t < IT; ++t) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (q0 + j < a.P) x[t][j] = ld_input_ordered(static_cast<const uint4*>(a.ptr.in[q0 + j]) + i0 + 32 * t);
        }
        // Item by item: the last batch's adds of item t, then its stores, so
        // that only one item's sum is live while the next one's loads land.
        const bool last = q0 + 8 >= a.P;
#pragma unroll
        for (int t = 0; t < IT; ++t) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (q0 + j < a.P) {
              if (q0 + j == 0) acc[t].template init_in<kQ8>(x[t][j]);
              else acc[t].template add_in<kQ8>(x[t][j]);
            }
          }
          if (last) {
            const uint4 v = acc[t].template round_out<kQ8>();
#pragma unroll
            for (int q = 0; q < kMaxP; ++q)
              if (q < a.P) st_stream(static_cast<uint4*>(a.ptr.out[q]) + i0 + 32 * t, v);
          }
        }
      }
    }
  }
  if (base < hi) {  // the one partial pass left to this CTA, if any
    const int64_t i0 = base + lane_off;
    for (int t = 0; t < IT; ++t) {
      const int64_t it = i0 + 32 * t;
      if (it < hi)
        store_item_rotated<D>(a.ptr.out, 0, a.P, c.r, it, a.n, reduce_item_out<D, kQ8>(a.ptr, 0, a.P, it, a.n));
    }
  }
  if (a.edge_sync) {
    __threadfence();
    block_barrier(a, c, kPhEnd);
  }
}

// 2-stage write mode, staged through shared memory with bulk copies. Same
// result and same work split by rank as k_twostage_write: rank r reduces slice
// r and streams it to all P outputs. The slice is cut into tiles of
// kStageItems items; CTA b of rank r takes tiles b, b+B, b+2B, ... A producer
// (lane 0 of warp 0) keeps up to `stages` tiles in flight: per tile, one bulk
// copy per input rank (kStageItems * 16 bytes) into a shared-memory stage, completing an
// mbarrier transaction count. Consumer warps (one thread per item) sum the P
// copies of their item from shared memory in ascending rank order, round once,
// and store the result to the P outputs, then free the stage for the producer.
// Loads of later tiles thus overlap stores of earlier ones without holding P
// vectors per thread in registers. A ragged last item (n not a multiple of the
// item size) is reduced from global memory by one thread.

constexpr int kStagedHeader = 512;   // mbarriers of up to kMaxStages stages
constexpr int kMaxStages = 24;

// Bounded mbarrier wait. Gives up when the time limit passes (recording a
// timeout) or when another thread of the CTA has given up (abort flag).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const KArgs& a, const Cta& c,
                                          volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > a.timeout_ns) {
        *abort_flag = 1;
        report_timeout(a, c, kPhCopy);
        return false;
      }
    }
  }
}

template <class D, int kStageItems, bool kQ8 = false>
__global__ void __launch_bounds__(32 + kStageItems) k_twostage_write_staged(const KArgs a) {
  constexpr uint32_t kStageTileBytes = kStageItems * 16;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // stages x 8 bytes, then stages x 8 bytes
  uint64_t* empty = full + a.stages;
  unsigned char* stage0 = smem + kStagedHeader;
  const int S = a.stages;
  const size_t stage_bytes = static_cast<size_t>(a.P) * kStageTileBytes;

  pdl_trigger();
  Cta c = cta_coords(a);
  const int64_t full_items = a.n / D::VE;  // items wholly inside the vector
  const int64_t piece = (a.items + a.P - 1) / a.P;
  const int64_t lo = lo_of(c.r, piece, a.items), hi = lo_of(c.r + 1, piece, a.items);
  const int64_t hi_full = hi < full_items ? hi : full_items;
  const int64_t rank_tiles = hi_full > lo ? (hi_full - lo + kStageItems - 1) / kStageItems : 0;
  const int64_t ntile = rank_tiles > c.b ? (rank_tiles - c.b + a.B - 1) / a.B : 0;
  auto tile_base = [&](int64_t k) { return lo + (c.b + k * a.B) * kStageItems; };

  if (threadIdx.x < a.P) {  // warm L2 with the first tiles while the previous call drains
    for (int64_t k = 0; k < ntile && k < S; ++k) {
      const int64_t base = tile_base(k);
      prefetch_items<D>(a.ptr.in[threadIdx.x], base, hi_full - base < kStageItems ? hi_full - base : kStageItems,
                        a.n);
    }
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kStageItems / 32);
    }
    s_abort = 0;
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();
  if (a.edge_sync) {
    cta_publish_flag(c, cta_take_ticket(a));
    if (!block_barrier(a, c, kPhStart)) return;  // no copy issued yet
  }
  volatile int* abort_flag = &s_abort;

  if (threadIdx.x == 0) {
    // Producer.
    int64_t issued = 0;
    for (int64_t k = 0; k < ntile; ++k) {
      const int st = static_cast<int>(k % S);
      if (k >= S && !mbar_wait(&empty[st], static_cast<uint32_t>((k / S) & 1) ^ 1u, a, c, abort_flag)) break;
      const int64_t base = tile_base(k);
      const uint32_t bytes =
          static_cast<uint32_t>((hi_full - base < kStageItems ? hi_full - base : kStageItems) * 16);
      mbar_arrive_expect_tx(&full[st], bytes * a.P);
      unsigned char* dst = stage0 + st * stage_bytes;
      for (int p = 0; p < a.P; ++p)
        bulk_load(dst + p * kStageTileBytes, static_cast<const unsigned char*>(a.ptr.in[p]) + base * 16, bytes,
                  &full[st]);
      issued = k + 1;
    }
    if (*abort_flag) {
      // Let the copies still in flight land before the CTA's shared memory goes away.
      for (int64_t k = issued > S ? issued - S : 0; k < issued; ++k) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[k % S], static_cast<uint32_t>((k / S) & 1)) &&
               globaltimer_ns() - t0 < a.timeout_ns) {
        }
      }
    }
  } else if (threadIdx.x >= 32) {
    // Consumers: thread i takes item i of every tile.
    const int ci = threadIdx.x - 32;
    for (int64_t k = 0; k < ntile; ++k) {
      const int st = static_cast<int>(k % S);
      bool ok = mbar_wait(&full[st], static_cast<uint32_t>((k / S) & 1), a, c, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int64_t base = tile_base(k);
      if (base + ci < hi_full) {
        const unsigned char* src = stage0 + st * stage_bytes + ci * 16;
        Acc<D> acc;
        acc.template init_in<kQ8>(ld_shared_v4(src));
        for (int p = 1; p < a.P; ++p) acc.template add_in<kQ8>(ld_shared_v4(src + p * kStageTileBytes));
        const uint4 v = acc.template round_out<kQ8>();
        for (int j = 0; j < a.P; ++j) {
          const int q = (c.r + j) % a.P;
          st_stream(static_cast<typename D::E*>(a.ptr.out[q]) + (base + ci) * D::VE, v);
        }
      }
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[st]);
    }
  }
  // Ragged last item, by the slice owner's first CTA.
  if (threadIdx.x == 32 && c.b == 0 && full_items < a.items && full_items >= lo && full_items < hi) {
    const uint4 v = reduce_item_out<D, kQ8>(a.ptr, 0, a.P, full_items, a.n);
    for (int p = 0; p < a.P; ++p) store_item<D, true>(a.ptr.out[p], full_items, a.n, v);
  }
  if (a.edge_sync) {
    __threadfence();
    block_barrier(a, c, kPhEnd);
  }
}

// 2-stage write mode [CAR "cross_device_reduce_2stage", write mode] with
// per-thread asynchronous copies. Same result and work split as
// k_twostage_write: thread i of CTA b (rank r) takes item i of tiles b, b+B,
// ... of slice r. For each tile it issues P 16-byte async copies (one per input
// rank) into its own shared-memory slots and keeps S tiles in flight; it then
// sums its P slots in ascending rank order, rounds once, and stores to all P
// outputs. A thread reads only slots it filled itself, so its own copy groups
// are the only synchronisation: no mbarrier, no producer lane, and all TI
// threads issue copies in parallel (the staged kernel's single producer lane
// issues P bulk copies per tile one after another, which is what limits it
// on small messages at many ranks). Shared memory: S * P * TI * 16 bytes.
//
// With kScatter the same kernel is the standalone reduce-scatter: rank r's
// slice is its chunk (n / P elements, a whole number of items) and the result
// goes to out[r] only, at the chunk's local offset. kQ8: inputs and reduced
// slice pass the fp8 wire.
template <class D, int TI, int S, bool kScatter = false, bool kQ8 = false>
__global__ void __launch_bounds__(TI) k_twostage_write_async(const KArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  pdl_trigger();
  Cta c = cta_coords(a);
  const int64_t full_items = a.n / D::VE;
  const int64_t piece = (a.items + a.P - 1) / a.P;
  const int64_t lo = lo_of(c.r, piece, a.items), hi = lo_of(c.r + 1, piece, a.items);
  const int64_t hi_full = hi < full_items ? hi : full_items;
  const int64_t rank_tiles = hi_full > lo ? (hi_full - lo + TI - 1) / TI : 0;
  const int64_t ntile = rank_tiles > c.b ? (rank_tiles - c.b + a.B - 1) / a.B : 0;
  auto tile_base = [&](int64_t k) { return lo + (c.b + k * a.B) * TI; };
  if (threadIdx.x < a.P) {
    for (int64_t k = 0; k < ntile && k < S; ++k) {
      const int64_t base = tile_base(k);
      prefetch_items<D>(a.ptr.in[threadIdx.x], base, hi_full - base < TI ? hi_full - base : TI, a.n);
    }
  }
  pdl_wait();
  if (a.edge_sync) {
    cta_publish_flag(c, cta_take_ticket(a));
    if (!block_barrier(a, c, kPhStart)) return;
  }
  const size_t stage_bytes = static_cast<size_t>(a.P) * TI * 16;
  unsigned char* mine = smem + threadIdx.x * 16;
  auto issue = [&](int64_t k) {
    if (k < ntile) {
      const int64_t it = tile_base(k) + threadIdx.x;
      if (it < hi_full) {
        unsigned char* dst = mine + (k % S) * stage_bytes;
        for (int p = 0; p < a.P; ++p)
          cp_async16(dst + p * (TI * 16), static_cast<const unsigned char*>(a.ptr.in[p]) + it * 16);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int k = 0; k < S - 1; ++k) issue(k);
  for (int64_t k = 0; k < ntile; ++k) {
    issue(k + S - 1);
    cp_async_wait<S - 1>();
    const int64_t it = tile_base(k) + threadIdx.x;
    if (it < hi_full) {
      const unsigned char* src = mine + (k % S) * stage_bytes;
      Acc<D> acc;
      acc.template init_in<kQ8>(ld_shared_v4(src));
      for (int p = 1; p < a.P; ++p) acc.template add_in<kQ8>(ld_shared_v4(src + p * (TI * 16)));
      const uint4 v = acc.template round_out<kQ8>();
      if (kScatter) {
        st_stream(static_cast<typename D::E*>(a.ptr.out[c.r]) + (it - lo) * D::VE, v);
      } else {
        for (int j = 0; j < a.P; ++j) {
          const int q = add_mod(c.r, j, a.P);
          st_stream(static_cast<typename D::E*>(a.ptr.out[q]) + it * D::VE, v);
        }
      }
    }
  }
  cp_async_wait<0>();
  if (!kScatter && threadIdx.x == 0 && c.b == 0 && full_items < a.items && full_items >= lo && full_items < hi) {
    const uint4 v = reduce_item_out<D, kQ8>(a.ptr, 0, a.P, full_items, a.n);
    for (int p = 0; p < a.P; ++p) store_item<D, true>(a.ptr.out[p], full_items, a.n, v);
  }
  if (a.edge_sync) {
    __threadfence();
    block_barrier(a, c, kPhEnd);
  }
}

// Recursive doubling with fused payload words [NVRAR phase 2, "Fused
// Payloads", "Chunked Non-blocking Communication", "Sequence-Number
// Synchronization"], over R = 2^steps ranks. The vector is cut into C chunks;
// each thread holds one item of every chunk. At step s it stores all C items
// (tagged with the call's sequence number) into the step-s receive slot of its
// partner rank XOR 2^s without waiting, then takes the partner's items from its
// own slot as they arrive and keeps rnd(own + partner).
//
// A call covers its items in rounds of B*T threads per rank (T = kThreads):
// in round t, thread t0 of a rank holds items k*per_chunk + t*B*T + t0. Every
// rank runs the same split, so a thread only ever exchanges with the thread
// at the same position in its partner rank.
//
// Payload slots. A slot is 32 bytes (one item as four 8-byte words). Rank q
// receives its step-s words in `slot_items` slots of slot set `set`, at
//   ll + (((set * P + q) * steps + s) * slot_items + slot) * 4 words.
// When the grid covers the message in one round (slot_sets == 1) the slot of
// an item is its index. Otherwise (slot_sets == 2) piece k of thread t0 uses
// slot k*B*T + t0 in every round, in slot set (round & 1): the slots are bound
// by the grid, not by the message, so they stay in L2 however long the
// message is. A slot is written again two rounds later, and only after its
// reader has read it: the writer q reaches round t+2 only after finishing
// round t+1, whose step s needed the reader p's round-(t+1) word, which p
// sends only after it has finished round t (and so read its round-t slot).
// The tag of round t is the call's flag with bit 31 set to bit 1 of t (rd_tag),
// so a word left from round t-2 never passes for round t's. No slot is ever
// cleared: a word belongs to this round only if its high half equals the tag.

// Tag of round `rnd` of a call with flag f (f < 2^31, never 0).
__device__ __forceinline__ uint32_t rd_tag(uint32_t f, int64_t rnd) {
  return f | (static_cast<uint32_t>((rnd >> 1) & 1) << 31);
}

// Slot of piece k of thread t0 (item idx) in a round, per the layout above.
__device__ __forceinline__ int64_t rd_slot(const KArgs& a, int k, int64_t idx, int64_t t0, int64_t stride) {
  return a.slot_sets == 1 ? idx : k * stride + t0;
}

// Partner of rank r at step s. Flat RD: r XOR 2^s. Hierarchical (r = g*L + l):
// the rank holding the same slice l in group g XOR 2^s.
template <bool kHier>
__device__ __forceinline__ int rd_partner(int r, int s, int L) {
  if (!kHier) return r ^ (1 << s);
  const int g = r / L, l = r % L;
  return (g ^ (1 << s)) * L + l;
}

template <class D, int C, bool kHier>
__device__ __forceinline__ bool rd_exchange(const KArgs& a, const Cta& c, uint4 (&v)[C], const int64_t (&slot)[C],
                                            const bool (&val)[C], int set, uint32_t tag) {
  const bool mute = (a.fault_mask >> c.r) & 1u;
  for (int s = 0; s < a.steps; ++s) {
    const int q = rd_partner<kHier>(c.r, s, a.L);
    uint64_t* dst = a.ll + ((static_cast<size_t>(set) * a.P + q) * a.steps + s) * a.slot_items * 4;
    const uint64_t* src = a.ll + ((static_cast<size_t>(set) * a.P + c.r) * a.steps + s) * a.slot_items * 4;
    if (!mute) {
#pragma unroll
      for (int k = 0; k < C; ++k)
        if (val[k]) send_item(dst + slot[k] * 4, v[k], tag);
    }
    // Poll all C slots together (one L2 round trip per attempt, not C), then
    // re-poll only the items whose four words do not all carry the tag yet.
    uint64_t w[C][4];
    uint32_t pending = 0;
#pragma unroll
    for (int k = 0; k < C; ++k) {
      if (val[k]) {
        ld_payload4(src + slot[k] * 4, w[k][0], w[k][1], w[k][2], w[k][3]);
        pending |= 1u << k;
      }
    }
    uint64_t t0 = 0;
    uint32_t it = 0;
    for (;; ++it) {
#pragma unroll
      for (int k = 0; k < C; ++k)
        if (((pending >> k) & 1u) && (w[k][0] >> 32) == tag && (w[k][1] >> 32) == tag && (w[k][2] >> 32) == tag &&
            (w[k][3] >> 32) == tag)
          pending &= ~(1u << k);
      if (!pending) break;
      if ((it & 15u) == 15u) {
        if (t0 == 0) t0 = globaltimer_ns();
        if (ld_relaxed(a.ctrl + kFailEpoch) == c.flag) {
          record_spins(a, it + 1, false);
          return false;
        }
        if (globaltimer_ns() - t0 > a.timeout_ns) {
          report_timeout(a, c, kPhPayload);
          record_spins(a, it + 1, true);
          return false;
        }
      }
#pragma unroll
      for (int k = 0; k < C; ++k)
        if ((pending >> k) & 1u) ld_payload4(src + slot[k] * 4, w[k][0], w[k][1], w[k][2], w[k][3]);
    }
    if (val[0]) record_spins(a, it + 1, false);  // one wait per step (the C pieces are polled together)
#pragma unroll
    for (int k = 0; k < C; ++k) {
      if (val[k]) {
        const uint4 peer = make_uint4(static_cast<uint32_t>(w[k][0]), static_cast<uint32_t>(w[k][1]),
                                      static_cast<uint32_t>(w[k][2]), static_cast<uint32_t>(w[k][3]));
        v[k] = add_round<D>(v[k], peer);
      }
    }
  }
  return true;
}

// L2 prefetch of the items CTA b of a rank reads in the round after the one
// at `base` (T items of each of the C chunks of [lo, lo + len)), issued by
// threads 0..C-1 while this round's exchange runs.
template <class D, int C>
__device__ __forceinline__ void prefetch_next_round(const void* in, int64_t lo, int64_t len, int64_t per_chunk,
                                                    int64_t base, int64_t stride, int b, int64_t n) {
  if (threadIdx.x < C) {
    const int64_t k = threadIdx.x;
    const int64_t first = base + stride + static_cast<int64_t>(b) * kThreads;
    const int64_t end = min((k + 1) * per_chunk, len) - k * per_chunk;
    if (first < end) prefetch_items<D>(in, lo + k * per_chunk + first, min(static_cast<int64_t>(kThreads), end - first), n);
  }
}

// kMinBlocks 2 limits registers to fit two CTAs per SM (64 per thread: at most
// two pieces per thread without spills), which the library launches for the
// element wire (more threads in flight per SM; measured faster).
template <class D, int C, int kMinBlocks = 1>
__global__ void __launch_bounds__(kThreads, kMinBlocks) k_rd(const KArgs a) {
  pdl_trigger();
  Cta c = cta_coords(a);
  const int64_t stride = static_cast<int64_t>(a.B) * kThreads;
  const int64_t t0 = static_cast<int64_t>(c.b) * kThreads + threadIdx.x;
  const int64_t per_chunk = (a.items + C - 1) / C;
  if (threadIdx.x < C) {
    const int64_t first = threadIdx.x * per_chunk + static_cast<int64_t>(c.b) * kThreads;
    const int64_t count = min(static_cast<int64_t>(kThreads), (threadIdx.x + 1) * per_chunk - first);
    prefetch_items<D>(a.ptr.in[c.r], first, count, a.n);
  }
  pdl_wait();
  const unsigned long long ticket = cta_take_ticket(a);
  bool ok = true;
  // The trip count is the same for every thread of the CTA (the flag is
  // published inside the first trip, after that trip's input loads issue).
  int64_t rnd = 0;
  for (int64_t base = 0; base < per_chunk; base += stride, ++rnd) {
    const int64_t j = base + t0;
    uint4 v[C];
    int64_t idx[C], slot[C];
    bool val[C];
#pragma unroll
    for (int k = 0; k < C; ++k) {
      idx[k] = k * per_chunk + j;
      slot[k] = rd_slot(a, k, idx[k], t0, stride);
      val[k] = ok && j < per_chunk && idx[k] < a.items;
      if (val[k]) v[k] = load_item_input<D>(a.ptr.in[c.r], idx[k], a.n);
    }
    if (base == 0) cta_publish_flag(c, ticket);
    if (!ok) continue;
    prefetch_next_round<D, C>(a.ptr.in[c.r], 0, a.items, per_chunk, base, stride, c.b, a.n);
    ok = rd_exchange<D, C, false>(a, c, v, slot, val, a.slot_sets == 1 ? 0 : static_cast<int>(rnd & 1),
                                  rd_tag(c.flag, rnd));
    if (ok) {
#pragma unroll
      for (int k = 0; k < C; ++k)
        if (val[k]) store_item<D, true>(a.ptr.out[c.r], idx[k], a.n, v[k]);
    }
  }
}

// Hierarchical all-reduce [NVRAR Methodology item 3, phases 1-3] with P = G*L
// ranks, rank r = g*L + l. Phase 1 (in-group reduce-scatter): rank (g, l)
// reduces slice l (ceil(items / L) items) over the L ranks of group g in
// ascending order, one rounding. Phase 2 (inter-group recursive doubling):
// log2 G steps of fused-payload exchange with partner (g XOR 2^s, l). Phase 3
// (in-group all-gather): rank (g, l) streams slice l into the outputs of all
// L ranks of group g. Slices are cut into C chunks, and payload slots laid out
// by round, as in k_rd (item indices are relative to the slice; partners hold
// the same slice). kMinBlocks 2 limits registers to fit two CTAs per SM (more
// threads in flight when a call needs several rounds over its items).
template <class D, int C, int kMinBlocks = 1>
__global__ void __launch_bounds__(kThreads, kMinBlocks) k_hier(const KArgs a) {
  pdl_trigger();
  Cta c = cta_coords(a);
  const int L = a.L, g = c.r / L, l = c.r % L;
  const int64_t stride = static_cast<int64_t>(a.B) * kThreads;
  const int64_t t0 = static_cast<int64_t>(c.b) * kThreads + threadIdx.x;
  const int64_t piece = (a.items + L - 1) / L;
  const int64_t lo = lo_of(l, piece, a.items), len = lo_of(l + 1, piece, a.items) - lo;
  const int64_t per_chunk = (len + C - 1) / C;
  if (threadIdx.x < L * C) {  // input rank g*L + (tid / C), chunk tid % C
    const int k = threadIdx.x % C;
    const int64_t first = k * per_chunk + static_cast<int64_t>(c.b) * kThreads;
    const int64_t count = min(static_cast<int64_t>(kThreads), min((k + 1) * per_chunk, len) - first);
    prefetch_items<D>(a.ptr.in[g * L + threadIdx.x / C], lo + first, count, a.n);
  }
  pdl_wait();
  const unsigned long long ticket = cta_take_ticket(a);
  bool ok = true;
  int64_t rnd = 0;
  for (int64_t base = 0; base < per_chunk; base += stride, ++rnd) {  // same trip count in the whole CTA
    const int64_t j = base + t0;
    uint4 v[C];
    int64_t idx[C], slot[C];
    bool val[C];
#pragma unroll
    for (int k = 0; k < C; ++k) {
      idx[k] = k * per_chunk + j;
      slot[k] = rd_slot(a, k, idx[k], t0, stride);
      val[k] = ok && j < per_chunk && idx[k] < len;
      if (val[k]) v[k] = reduce_item<D>(a.ptr, g * L, L, lo + idx[k], a.n);
    }
    if (base == 0) cta_publish_flag(c, ticket);
    if (!ok) continue;
    // The next round reads the same items of all L inputs of the group: warm
    // L2 with them while this round's exchange runs (threads 0..L*C-1, one
    // input and chunk each), when the host asks for it (prefetch_next).
    if (a.prefetch_next && threadIdx.x < L * C) {
      const int64_t k = threadIdx.x % C;
      const int64_t first = base + stride + static_cast<int64_t>(c.b) * kThreads;
      const int64_t end = min((k + 1) * per_chunk, len) - k * per_chunk;
      if (first < end)
        prefetch_items<D>(a.ptr.in[g * L + threadIdx.x / C], lo + k * per_chunk + first,
                          min(static_cast<int64_t>(kThreads), end - first), a.n);
    }
    ok = rd_exchange<D, C, true>(a, c, v, slot, val, a.slot_sets == 1 ? 0 : static_cast<int>(rnd & 1),
                                 rd_tag(c.flag, rnd));
    if (ok) {
#pragma unroll
      for (int k = 0; k < C; ++k)
        if (val[k]) store_item_rotated<D>(a.ptr.out, g * L, L, l, lo + idx[k], a.n, v[k]);
    }
  }
}

// Recursive doubling and the hierarchical all-reduce with fp32 partials on
// the wire (16-bit element types). Each 16-byte input item becomes two fp32
// quads that travel as fused payload words exactly like fp32 elements (so
// twice the payload words of the element-type wire); the steps add in fp32
// without rounding, and the store rounds once to the element type. A slot of
// the element wire becomes two quad slots (2 * slot, 2 * slot + 1); the host
// doubles slot_items. C is at most 2 here (2C quads in flight per thread); the
// library runs k_rd_wide with one piece and two CTAs per SM (kMinBlocks 2).
template <class D, int C, int kMinBlocks = 1>
__global__ void __launch_bounds__(kThreads, kMinBlocks) k_rd_wide(const KArgs a) {
  pdl_trigger();
  Cta c = cta_coords(a);
  const int64_t stride = static_cast<int64_t>(a.B) * kThreads;
  const int64_t t0 = static_cast<int64_t>(c.b) * kThreads + threadIdx.x;
  const int64_t per_chunk = (a.items + C - 1) / C;
  if (threadIdx.x < C) {
    const int64_t first = threadIdx.x * per_chunk + static_cast<int64_t>(c.b) * kThreads;
    const int64_t count = min(static_cast<int64_t>(kThreads), (threadIdx.x + 1) * per_chunk - first);
    prefetch_items<D>(a.ptr.in[c.r], first, count, a.n);
  }
  pdl_wait();
  const unsigned long long ticket = cta_take_ticket(a);
  bool ok = true;
  int64_t rnd = 0;
  for (int64_t base = 0; base < per_chunk; base += stride, ++rnd) {  // same trip count in the whole CTA
    const int64_t j = base + t0;
    uint4 q[2 * C];
    int64_t qslot[2 * C], idx[C];
    bool qval[2 * C];
#pragma unroll
    for (int k = 0; k < C; ++k) {
      idx[k] = k * per_chunk + j;
      const bool val = ok && j < per_chunk && idx[k] < a.items;
      const int64_t sl = rd_slot(a, k, idx[k], t0, stride);
      qslot[2 * k] = 2 * sl;
      qslot[2 * k + 1] = 2 * sl + 1;
      qval[2 * k] = qval[2 * k + 1] = val;
      if (val) {
        Acc<D> x;
        x.init(load_item_input<D>(a.ptr.in[c.r], idx[k], a.n));
        floats_to_quads(x.v, q[2 * k], q[2 * k + 1]);
      }
    }
    if (base == 0) cta_publish_flag(c, ticket);
    if (!ok) continue;
    prefetch_next_round<D, C>(a.ptr.in[c.r], 0, a.items, per_chunk, base, stride, c.b, a.n);
    ok = rd_exchange<F32T, 2 * C, false>(a, c, q, qslot, qval, a.slot_sets == 1 ? 0 : static_cast<int>(rnd & 1),
                                         rd_tag(c.flag, rnd));
    if (ok) {
#pragma unroll
      for (int k = 0; k < C; ++k)
        if (qval[2 * k]) store_item<D, true>(a.ptr.out[c.r], idx[k], a.n, quads_to_item<D>(q[2 * k], q[2 * k + 1]));
    }
  }
}

template <class D, int C>
__global__ void __launch_bounds__(kThreads) k_hier_wide(const KArgs a) {
  pdl_trigger();
  Cta c = cta_coords(a);
  const int L = a.L, g = c.r / L, l = c.r % L;
  const int64_t stride = static_cast<int64_t>(a.B) * kThreads;
  const int64_t t0 = static_cast<int64_t>(c.b) * kThreads + threadIdx.x;
  const int64_t piece = (a.items + L - 1) / L;
  const int64_t lo = lo_of(l, piece, a.items), len = lo_of(l + 1, piece, a.items) - lo;
  const int64_t per_chunk = (len + C - 1) / C;
  if (threadIdx.x < L * C) {
    const int k = threadIdx.x % C;
    const int64_t first = k * per_chunk + static_cast<int64_t>(c.b) * kThreads;
    const int64_t count = min(static_cast<int64_t>(kThreads), min((k + 1) * per_chunk, len) - first);
    prefetch_items<D>(a.ptr.in[g * L + threadIdx.x / C], lo + first, count, a.n);
  }
  pdl_wait();
  const unsigned long long ticket = cta_take_ticket(a);
  bool ok = true;
  int64_t rnd = 0;
  for (int64_t base = 0; base < per_chunk; base += stride, ++rnd) {  // same trip count in the whole CTA
    const int64_t j = base + t0;
    uint4 q[2 * C];
    int64_t qslot[2 * C], idx[C];
    bool qval[2 * C];
#pragma unroll
    for (int k = 0; k < C; ++k) {
      idx[k] = k * per_chunk + j;
      const bool val = ok && j < per_chunk && idx[k] < len;
      const int64_t sl = rd_slot(a, k, idx[k], t0, stride);
      qslot[2 * k] = 2 * sl;
      qslot[2 * k + 1] = 2 * sl + 1;
      qval[2 * k] = qval[2 * k + 1] = val;
      if (val) {
        const Acc<D> s = reduce_item_acc<D>(a.ptr, g * L, L, lo + idx[k], a.n);  // not rounded
        floats_to_quads(s.v, q[2 * k], q[2 * k + 1]);
      }
    }
    if (base == 0) cta_publish_flag(c, ticket);
    if (!ok) continue;
    ok = rd_exchange<F32T, 2 * C, true>(a, c, q, qslot, qval, a.slot_sets == 1 ? 0 : static_cast<int>(rnd & 1),
                                        rd_tag(c.flag, rnd));
    if (ok) {
#pragma unroll
      for (int k = 0; k < C; ++k) {
        if (!qval[2 * k]) continue;
        store_item_rotated<D>(a.ptr.out, g * L, L, l, lo + idx[k], a.n, quads_to_item<D>(q[2 * k], q[2 * k + 1]));
      }
    }
  }
}

// Standalone reduce-scatter [NVRAR phase 1 over one group]: rank p writes
// elements [p*m, (p+1)*m) of the ascending-rank sum into out[p], m = n / P.
// Needs no flags. 16-byte path when m is a multiple of the item size (so
// every slice starts on a 16-byte boundary), element path otherwise. Up to
// 1 MiB per rank the async-copy write kernel in its scatter form is used
// instead of the 16-byte path here.
template <class D>
__global__ void __launch_bounds__(kThreads, 2) k_reduce_scatter(const KArgs a) {
  pdl_trigger();
  const int r = static_cast<int>(blockIdx.x % a.P), b = static_cast<int>(blockIdx.x / a.P);
  const int64_t stride = static_cast<int64_t>(a.B) * kThreads;
  const int64_t t0 = static_cast<int64_t>(b) * kThreads + threadIdx.x;
  const int64_t m = a.n / a.P;
  if (m % D::VE == 0 && threadIdx.x < a.P) {
    const int64_t mi = m / D::VE, first = static_cast<int64_t>(b) * kThreads;
    const int64_t count = min(static_cast<int64_t>(kThreads), mi - first);
    prefetch_items<D>(a.ptr.in[threadIdx.x], r * mi + first, count, a.n);
  }
  pdl_wait();
  if (m % D::VE == 0) {
    const int64_t mi = m / D::VE;
    for (int64_t j = t0; j < mi; j += stride)
      store_item<D, true>(a.ptr.out[r], j, m, reduce_item<D>(a.ptr, 0, a.P, r * mi + j, a.n));
  } else {
    using E = typename D::E;
    for (int64_t e = t0; e < m; e += stride) {
      const int64_t src = r * m + e;
      float acc = D::elem_to_f(static_cast<const E*>(a.ptr.in[0])[src]);
      for (int q = 1; q < a.P; ++q) acc = __fadd_rn(acc, D::elem_to_f(static_cast<const E*>(a.ptr.in[q])[src]));
      static_cast<E*>(a.ptr.out[r])[e] = D::f_to_elem(acc);
    }
  }
}

// Standalone all-gather [NVRAR phase 3 over one group], push form: rank s
// reads its n/P elements and streams them to offset s*m of all P outputs.
// The P destinations are split over G = a.chunks groups of CTAs (group g
// writes outputs g, g+G, g+2G, ...), so that a short slice still spreads over
// many SMs; each group reads the slice once more, from L2.
template <class D>
__global__ void __launch_bounds__(kThreads, 2) k_all_gather(const KArgs a) {
  pdl_trigger();
  const int s = static_cast<int>(blockIdx.x % a.P);
  const int rest = static_cast<int>(blockIdx.x / a.P);
  const int b = rest % a.B, g = rest / a.B, G = a.chunks;
  const int64_t stride = static_cast<int64_t>(a.B) * kThreads;
  const int64_t t0 = static_cast<int64_t>(b) * kThreads + threadIdx.x;
  const int64_t m = a.n / a.P;
  if (m % D::VE == 0 && threadIdx.x == 0 && g == 0)
    prefetch_items<D>(a.ptr.in[s], static_cast<int64_t>(b) * kThreads, kThreads, m);
  pdl_wait();
  if (m % D::VE == 0) {
    const int64_t mi = m / D::VE;
    for (int64_t j = t0; j < mi; j += stride) {
      const uint4 v = load_item_input<D>(a.ptr.in[s], j, m);
      for (int q = g; q < a.P; q += G) store_item<D, true>(a.ptr.out[q], s * mi + j, a.n, v);
    }
  } else {
    using E = typename D::E;
    for (int64_t e = t0; e < m; e += stride) {
      const E v = static_cast<const E*>(a.ptr.in[s])[e];
      for (int q = g; q < a.P; q += G) static_cast<E*>(a.ptr.out[q])[s * m + e] = v;
    }
  }
}

}  // namespace vrar
