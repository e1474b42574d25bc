// Host-thread model of the virtual-rank synchronisation protocol.
//
// Test infrastructure, independent of the CUDA sources (nothing is included
// from them): it restates in C++ atomics the protocol the kernels follow, with
// one std::thread per CTA, so that the protocol logic can be exercised for
// races (under ThreadSanitizer) and for a missing rank without a GPU.
//
// The protocol, as the kernels implement it from [CAR] "Summary" / "Root
// cause" (start, mid and end flag barriers polled with acquire loads) and
// [NVRAR] "Fused Payloads" / "Sequence-Number Synchronization" (data and
// sequence number in one 8-byte word, no separate signal):
//  * one 64-bit ticket per device: every CTA of a call adds 1; the CTA that
//    brings the low half to the grid size also adds 2^32 - grid, so the high
//    half counts calls and the low half returns to 0. A CTA's flag for the
//    call is (high half before its add) mod (2^31 - 1) + 1: never 0, below 2^31.
//  * a barrier: CTA (r, b) stores the flag into word [(p*B + b)*32 + r] of the
//    phase's array for every rank p (release), then waits until word
//    [(r*B + b)*32 + p] equals the flag for every p (acquire). Words are never
//    cleared; equality with a flag that only grows rejects every stale word.
//  * recursive doubling in rounds: a rank's items are cut into C chunks and
//    covered by S = B * T thread positions per round (T per CTA); in round t
//    position t0 holds item k*per_chunk + t*S + t0 of every chunk k. At step s
//    rank r stores {data | tag << 32} into the step-s slot of partner
//    r XOR 2^s and polls its own step-s slot until the high half equals the
//    tag, then adds. With one round the slot of an item is its index; with
//    several, piece k of position t0 uses slot k*S + t0 of slot set (t & 1),
//    and the tag of round t is the flag with bit 31 set to bit 1 of t. A slot
//    is rewritten two rounds later only after its reader has read it (the
//    writer needs the reader's next-round word first), and the lap bit keeps
//    a word from two rounds back from passing for the current one.
//  * every wait is bounded; the first CTA to give up records a status and the
//    call's flag as the failed epoch, and every other wait of that call stops
//    as soon as it sees the epoch.
//
// Checks: thousands of back-to-back calls whose shape (P, B, items, C)
// changes from call to call, many of them several rounds long, with one rank
// per call held back (before its first poll, and before its sends two rounds
// later), each with exact integer sums on every rank from both the
// recursive doubling and the pull 2-stage (a stale or early word, or a read
// that the mid barrier did not order after its write, would change them; one
// rank per call writes its 2-stage slice late, and under ThreadSanitizer the
// plain 2-stage data must be ordered by the barrier's release and acquire); one call in which a rank never posts, which
// must end with the status set and every thread returned; and the calls after
// it, which must be correct again. Prints "ok" and exits 0, else exits 1.
#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <thread>
#include <vector>

// Planted mistakes for the tests (0 = the protocol as specified): 1 the
// payload poll ignores the sequence number; 2 the ticket's last arriver does
// not return the low half to 0 (every call then has the same flag); 3 a
// barrier posts into the waiter's own words instead of the peers'; 4 the
// rounds of a call share one slot set; 5 round tags carry no lap bit.
#ifndef MODEL_MUTANT
#define MODEL_MUTANT 0
#endif

namespace {

constexpr int kMaxP = 32;
constexpr int kMaxB = 4;
constexpr int kPhases = 3;  // start, mid, end
constexpr int kMaxSteps = 5;
constexpr int kMaxItems = 64;  // items per rank
constexpr int kT = 2;          // thread positions per CTA in the recursive doubling
// Waits are bounded by time, as on the device (where the limit is 2 s by
// default and read from %globaltimer); a poll count would give up on a peer
// thread that the OS has simply not scheduled yet.
constexpr std::chrono::milliseconds kWaitLimit{1000};

struct Device {
  std::atomic<uint64_t> ticket{0};
  std::atomic<uint32_t> status{0};
  std::atomic<uint32_t> fail_epoch{0};
  std::vector<std::atomic<uint32_t>> sig;
  std::vector<std::atomic<uint64_t>> ll;
  Device() : sig(kPhases * kMaxB * kMaxP * kMaxP), ll(2 * kMaxP * kMaxSteps * kMaxItems) {
    for (auto& w : sig) w.store(0);
    for (auto& w : ll) w.store(0);
  }
};

struct Call {
  int P, B, items, steps, C;
  int muted;  // rank that never posts or sends, -1 for none
  std::vector<int32_t> in, out;  // [P][items]; out: recursive doubling's result
  std::vector<int32_t> pull;     // [P][items]: the pull 2-stage's result (plain, not atomic)
  int late;                      // rank whose 2-stage phase 1 starts late
};

uint32_t take_flag(Device& d, int grid) {
  const uint64_t old = d.ticket.fetch_add(1, std::memory_order_acq_rel);
  if (MODEL_MUTANT != 2 && static_cast<uint32_t>(old) == static_cast<uint32_t>(grid - 1))
    d.ticket.fetch_add((uint64_t{1} << 32) - static_cast<uint64_t>(grid), std::memory_order_acq_rel);
  return static_cast<uint32_t>(old >> 32) % 0x7FFFFFFFu + 1u;
}

// Bounded wait for `word == flag`; false once the limit passes or the call's
// epoch is marked failed.
template <class W, class Match>
bool wait_for(Device& d, W& word, uint32_t flag, Match match) {
  const auto t0 = std::chrono::steady_clock::now();
  for (long it = 0;; ++it) {
    if (match(word.load(std::memory_order_acquire))) return true;
    if ((it & 63) == 63) {
      if (d.fail_epoch.load(std::memory_order_relaxed) == flag) return false;
      if (std::chrono::steady_clock::now() - t0 > kWaitLimit) {
        uint32_t zero = 0;
        d.status.compare_exchange_strong(zero, 1);
        d.fail_epoch.store(flag, std::memory_order_relaxed);
        return false;
      }
      std::this_thread::yield();
    }
  }
}

bool barrier(Device& d, const Call& c, int phase, int r, int b, uint32_t flag) {
  std::atomic<uint32_t>* sig = &d.sig[static_cast<size_t>(phase) * kMaxB * kMaxP * kMaxP];
  if (r != c.muted)
    for (int p = 0; p < c.P; ++p)
      sig[MODEL_MUTANT == 3 ? (r * c.B + b) * kMaxP + p : (p * c.B + b) * kMaxP + r].store(flag, std::memory_order_release);
  for (int p = 0; p < c.P; ++p)
    if (!wait_for(d, sig[(r * c.B + b) * kMaxP + p], flag, [&](uint32_t w) { return w == flag; })) return false;
  return true;
}

// CTA (r, b): start barrier; recursive doubling over its thread positions
// b*kT .. b*kT + kT - 1, round by round; the pull 2-stage on the items b, b+B,
// ... (phase 1: rank r sums its slice into pull[r]; mid barrier; phase 2: it
// copies every other slice s out of pull[s]); store; end barrier.
void cta(Device& d, Call& c, int r, int b) {
  const uint32_t flag = take_flag(d, c.P * c.B);
  if (!barrier(d, c, 0, r, b, flag)) return;
  const int S = c.B * kT;
  const int per_chunk = (c.items + c.C - 1) / c.C;
  const int rounds = (per_chunk + S - 1) / S;
  const bool reuse = rounds > 1;
  for (int rnd = 0, base = 0; base < per_chunk; base += S, ++rnd) {
    const int set = (reuse && MODEL_MUTANT != 4) ? (rnd & 1) : 0;
    const uint32_t tag = MODEL_MUTANT == 5 ? flag : flag | (static_cast<uint32_t>((rnd >> 1) & 1) << 31);
    int idx[kT][8], slot[kT][8];
    bool val[kT][8];
    int32_t v[kT][8];
    for (int u = 0; u < kT; ++u) {
      const int t0 = b * kT + u, j = base + t0;
      for (int k = 0; k < c.C; ++k) {
        idx[u][k] = k * per_chunk + j;
        slot[u][k] = reuse ? k * S + t0 : idx[u][k];
        val[u][k] = j < per_chunk && idx[u][k] < c.items;
        v[u][k] = val[u][k] ? c.in[r * c.items + idx[u][k]] : 0;
      }
    }
    for (int s = 0; s < c.steps; ++s) {
      const int q = r ^ (1 << s);
      std::atomic<uint64_t>* dst = &d.ll[((static_cast<size_t>(set) * kMaxP + q) * kMaxSteps + s) * kMaxItems];
      std::atomic<uint64_t>* src = &d.ll[((static_cast<size_t>(set) * kMaxP + r) * kMaxSteps + s) * kMaxItems];
      if (r == c.late && rnd == 2 && s == 0) std::this_thread::sleep_for(std::chrono::microseconds(200));
      if (r != c.muted)
        for (int u = 0; u < kT; ++u)
          for (int k = 0; k < c.C; ++k)
            if (val[u][k])
              dst[slot[u][k]].store((static_cast<uint64_t>(tag) << 32) | static_cast<uint32_t>(v[u][k]),
                                    std::memory_order_release);
      if (r == c.late && rnd == 0 && s == 0) std::this_thread::sleep_for(std::chrono::microseconds(200));
      for (int u = 0; u < kT; ++u)
        for (int k = 0; k < c.C; ++k) {
          if (!val[u][k]) continue;
          auto& w = src[slot[u][k]];
          uint64_t got = 0;
          if (!wait_for(d, w, flag, [&](uint64_t x) {
                got = x;
                return MODEL_MUTANT == 1 || static_cast<uint32_t>(x >> 32) == tag;
              }))
            return;
          v[u][k] += static_cast<int32_t>(static_cast<uint32_t>(got));
        }
    }
    for (int u = 0; u < kT; ++u)
      for (int k = 0; k < c.C; ++k)
        if (val[u][k]) c.out[r * c.items + idx[u][k]] = v[u][k];
  }
  const int piece = (c.items + c.P - 1) / c.P;
  auto slice_lo = [&](int s) { return s * piece < c.items ? s * piece : c.items; };
  if (r == c.late) std::this_thread::sleep_for(std::chrono::microseconds(300));
  for (int i = slice_lo(r); i < slice_lo(r + 1); ++i) {
    if (i % c.B != b) continue;
    int32_t acc = 0;
    for (int p = 0; p < c.P; ++p) acc += c.in[p * c.items + i];
    c.pull[r * c.items + i] = acc;
  }
  if (!barrier(d, c, 1, r, b, flag)) return;
  for (int s = 0; s < c.P; ++s) {
    if (s == r) continue;
    for (int i = slice_lo(s); i < slice_lo(s + 1); ++i)
      if (i % c.B == b) c.pull[r * c.items + i] = c.pull[s * c.items + i];
  }
  barrier(d, c, 2, r, b, flag);
}

void run(Device& d, Call& c) {
  std::vector<std::thread> ts;
  for (int b = 0; b < c.B; ++b)
    for (int r = 0; r < c.P; ++r) ts.emplace_back(cta, std::ref(d), std::ref(c), r, b);
  for (auto& t : ts) t.join();  // the next call starts after this one: stream order
}

Call make_call(int k, int P, int B, int items, int C, int muted) {
  Call c{P, B, items, 0, C, muted, std::vector<int32_t>(P * items), std::vector<int32_t>(P * items, 0),
         std::vector<int32_t>(P * items, 0), k % P};
  while ((1 << c.steps) < P) ++c.steps;
  for (int p = 0; p < P; ++p)
    for (int i = 0; i < items; ++i) c.in[p * items + i] = ((7 * p + i + 3 * k) % 17) - 8 + 100 * (k % 7);
  return c;
}

bool exact(const Call& c) {
  for (int i = 0; i < c.items; ++i) {
    int32_t want = 0;
    for (int p = 0; p < c.P; ++p) want += c.in[p * c.items + i];
    for (int p = 0; p < c.P; ++p)
      if (c.out[p * c.items + i] != want || c.pull[p * c.items + i] != want) return false;
  }
  return true;
}

}  // namespace

int main(int argc, char** argv) {
  const int calls = argc > 1 ? std::atoi(argv[1]) : 3000;
  Device d;
  // {P, B, items, C}: one-round and many-round calls (up to 32 rounds).
  constexpr int kShapes = 10;
  const int shapes[kShapes][4] = {{2, 1, 5, 1},  {4, 2, 17, 2}, {8, 1, 33, 1}, {8, 4, 64, 2}, {16, 2, 9, 1},
                                  {32, 1, 3, 1}, {4, 4, 1, 3},  {2, 1, 64, 1}, {4, 1, 60, 3}, {8, 2, 64, 3}};
  for (int k = 0; k < calls; ++k) {
    const auto& sh = shapes[k % kShapes];
    Call c = make_call(k, sh[0], sh[1], sh[2], sh[3], -1);
    run(d, c);
    if (d.status.load() != 0 || !exact(c)) {
      std::fprintf(stderr, "call %d (P=%d B=%d items=%d C=%d): status %u, exact %d\n", k, c.P, c.B, c.items, c.C,
                   d.status.load(), exact(c) ? 1 : 0);
      return 1;
    }
  }
  // A rank that never posts or sends: every wait of the call gives up, the
  // status is recorded, every thread returns.
  Call bad = make_call(calls, 8, 2, 20, 2, 3);
  run(d, bad);
  if (d.status.load() != 1) {
    std::fprintf(stderr, "missing rank: status %u\n", d.status.load());
    return 1;
  }
  d.status.store(0);  // the host reads and clears it
  // Later calls are correct again: their flags are new, so no word written in
  // the failed call (or before it) can match.
  for (int k = calls + 1; k < calls + 50; ++k) {
    const auto& sh = shapes[k % kShapes];
    Call c = make_call(k, sh[0], sh[1], sh[2], sh[3], -1);
    run(d, c);
    if (d.status.load() != 0 || !exact(c)) {
      std::fprintf(stderr, "after the failure, call %d: status %u, exact %d\n", k, d.status.load(), exact(c) ? 1 : 0);
      return 1;
    }
  }
  const uint64_t t = d.ticket.load();
  if (static_cast<uint32_t>(t) != 0 || (t >> 32) != static_cast<uint64_t>(calls + 50)) {
    std::fprintf(stderr, "ticket %llx after %d calls\n", static_cast<unsigned long long>(t), calls + 50);
    return 1;
  }
  std::printf("ok\n");
  return 0;
}
