/*
 * CPU oracle for the virtual-rank all-reduce.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it. It shares no code, header, table or
 * constant with the CUDA library: it is a plain, slow, single-threaded
 * restatement of what each algorithm computes, written so that a reader can
 * check it against the sources by eye.
 *
 * Sources (web pages; sections as printed on them):
 *  [NVRAR]  "Technical Summary: Understanding and Improving Communication
 *           Performance in Multi-node LLM Inference" (gist.science summary of
 *           arXiv 2511.09557), section "Methodology", item 3 "Proposed Solution
 *           (NVRAR)": three phases (intra-node reduce-scatter, inter-node
 *           recursive doubling, intra-node all-gather) and the optimisations
 *           "Chunked Non-blocking Communication", "Fused Payloads",
 *           "Sequence-Number Synchronization".
 *  [CAR]    "fix(custom_all_reduce): use SYSTEM scope + ACQUIRE ordering for
 *           cross-device signal loads" (ROCm/aiter pull request 4786),
 *           sections "Summary" and "Root cause": the custom all-reduce with
 *           start/end flag barriers, the 2-stage (reduce-scatter + all-gather)
 *           kernel and its write mode, which stores the reduced slice straight
 *           into every rank's registered output.
 *
 * Numerics (readings of the sources, which fix none of this):
 *  - Inputs are bf16, fp16 (IEEE binary16) or fp32. Every add is one IEEE-754
 *    binary32 add with round-to-nearest-even; a 16-bit operand is widened
 *    exactly to fp32 first.
 *  - A reduction of several ranks' values adds them left to right in
 *    ascending rank order starting from rank 0, and rounds once to the tensor
 *    type at the end.
 *  - Recursive doubling moves values in the tensor type: each step adds two
 *    tensor-typed values in fp32 and rounds back to the tensor type. The
 *    "fp32 wire" variants ("rd_fp32wire", "hier_fp32wire") move fp32 partials
 *    instead: no rounding until the final store (the other reading of what a
 *    fused payload word carries).
 *  - fp32 -> bf16 is round-to-nearest-even from the definition of the format
 *    (bf16 = the upper 16 bits of a binary32); any NaN becomes 0x7FC0.
 *  - fp32 -> fp16 is round-to-nearest-even from the definition of binary16
 *    (1 sign, 5 exponent bits biased by 15, 10 fraction bits; subnormals in
 *    steps of 2^-24; values from 65520 up round to infinity); NaN -> 0x7E00.
 *
 *  - fp8 payloads ("oneshot_fp8", "twostage_fp8", "twostage_write_fp8"; the
 *    ca_fp8_quant flag of the custom all-reduce, whose scheme the sources do
 *    not give - this is the reading taken): every value that passes from one
 *    rank to another travels as OCP FP8 E4M3 (1 sign, 4 exponent bits biased
 *    by 7, 3 fraction bits, subnormals in steps of 2^-9, no infinities,
 *    largest finite 448) with one binary32 scale per group of 8 consecutive
 *    elements (one 16-byte item of a 16-bit tensor; the last group holds what
 *    is left). The scale is s = amax / 448 (amax = the largest magnitude in the
 *    group; s = 1 if that division gives 0); an element quantises to
 *    q = E4M3(x / s), round to nearest even, magnitudes past 448 saturating to
 *    448, and dequantises to q * s (binary32 division and product, both round
 *    to nearest even). One-shot quantises every input once (every rank reads
 *    all P inputs through the fp8 wire, its own included, so that all outputs
 *    agree); the 2-stage variants quantise the inputs for the reduce-scatter
 *    and the reduced binary32 slice again for the all-gather, and every rank,
 *    the owner included, stores the dequantised value rounded to the tensor
 *    type. A group whose binary32 sum is infinite has an infinite scale in
 *    that second quantisation, so all its values come back as NaN.
 *
 * Floating-point environment: the functions below clear the x86 flush-to-zero
 * and denormals-are-zero bits for their duration, so subnormal inputs and
 * sums are handled exactly as IEEE-754 says, whatever the caller left set.
 */

#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <vector>

#if defined(__SSE__) || defined(__x86_64__)
#include <xmmintrin.h>
#define ORACLE_HAVE_MXCSR 1
#endif

namespace {

/* ---- floating-point environment ------------------------------------------------ */

struct IeeeScope {
#ifdef ORACLE_HAVE_MXCSR
    unsigned saved;
    IeeeScope() : saved(_mm_getcsr()) { _mm_setcsr(saved & ~0x8040u); /* FTZ | DAZ */ }
    ~IeeeScope() { _mm_setcsr(saved); }
#endif
};

/* ---- bf16 <-> fp32 from the format's definition --------------------------------- */

inline float bits_to_f32(uint32_t u) {
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

inline uint32_t f32_to_bits(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return u;
}

/* A bf16 value is the high half of a binary32, so widening appends 16 zero bits. */
inline float bf16_widen(uint16_t h) { return bits_to_f32(static_cast<uint32_t>(h) << 16); }

/* Round a binary32 to the nearest bf16, ties to even. Adding 0x7FFF plus the
 * lowest kept bit to the full pattern carries into the kept half exactly when
 * the dropped half is above one half ulp, or equal to it with an odd kept half.
 * The carry out of the mantissa steps the exponent, which also turns the
 * largest finite values that round up into infinity, as the format requires. */
inline uint16_t bf16_round(float f) {
    uint32_t u = f32_to_bits(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0u) return 0x7FC0u;
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7FFFu + keep_lsb;
    return static_cast<uint16_t>(u >> 16);
}

/* binary16 -> binary32, exact. Subnormal halves are fraction * 2^-24 (a
 * product of an integer below 1024 and a power of two: exact in binary32). */
inline float half_widen(uint16_t h) {
    const uint32_t sign = static_cast<uint32_t>(h & 0x8000u) << 16;
    const uint32_t exp = (h >> 10) & 0x1Fu, frac = h & 0x3FFu;
    if (exp == 0) {
        const float v = static_cast<float>(frac) * (1.0f / 16777216.0f);
        return sign ? -v : v;
    }
    if (exp == 31) return bits_to_f32(sign | 0x7F800000u | (frac << 13));
    return bits_to_f32(sign | ((exp + 112u) << 23) | (frac << 13));
}

/* binary32 -> binary16, round to nearest, ties to even. */
inline uint16_t half_round(float f) {
    const uint32_t u = f32_to_bits(f);
    const uint16_t sign = static_cast<uint16_t>((u >> 16) & 0x8000u);
    const uint32_t a = u & 0x7FFFFFFFu;
    if (a > 0x7F800000u) return 0x7E00u;                        // NaN
    if (a >= 0x477FF000u) return static_cast<uint16_t>(sign | 0x7C00u);  // >= 65520 (and inf) -> inf
    if (a >= 0x38800000u) {                                     // >= 2^-14: a normal half
        const uint32_t m = a - 0x38000000u;                     // exponent rebias 127 -> 15
        uint32_t keep = m >> 13;
        const uint32_t rest = m & 0x1FFFu;
        if (rest > 0x1000u || (rest == 0x1000u && (keep & 1u))) keep += 1;  // a carry may step the exponent
        return static_cast<uint16_t>(sign | keep);
    }
    // Subnormal (or zero) half: round |f| / 2^-24 to an integer, ties to even.
    // The scaling by a power of two is exact, and so is the fraction below.
    const float q = bits_to_f32(a) * 16777216.0f;
    uint32_t i = static_cast<uint32_t>(q);
    const float rest = q - static_cast<float>(i);
    if (rest > 0.5f || (rest == 0.5f && (i & 1u))) i += 1;     // i may reach 1024 = the smallest normal
    return static_cast<uint16_t>(sign | i);
}

/* ---- element types ------------------------------------------------------------ */

struct Bf16 {
    using T = uint16_t;
    static float widen(T v) { return bf16_widen(v); }
    static T narrow(float a) { return bf16_round(a); }
    static constexpr int64_t bytes = 2;
};

struct F16 {
    using T = uint16_t;
    static float widen(T v) { return half_widen(v); }
    static T narrow(float a) { return half_round(a); }
    static constexpr int64_t bytes = 2;
};

struct F32 {
    using T = float;
    static float widen(T v) { return v; }
    static T narrow(float a) { return a; }
    static constexpr int64_t bytes = 4;
};

/* The one binary32 add every algorithm uses. volatile keeps the compiler from
 * fusing or reassociating it (the build also passes -ffp-contract=off). */
inline float add32(float a, float b) {
    volatile float s = a + b;
    return s;
}

/* Owner split used by the 2-stage and hierarchical phases: `parts` contiguous
 * pieces of ceil(n / (parts * V)) * V elements, V = elements per 16 bytes; the
 * last pieces may be short or empty. (Values do not depend on this split.) */
struct Split {
    int64_t piece;
    int64_t n;
    Split(int64_t n_, int parts, int64_t esize) : n(n_) {
        int64_t V = 16 / esize;
        int64_t per = (n + static_cast<int64_t>(parts) * V - 1) / (static_cast<int64_t>(parts) * V);
        piece = per * V;
    }
    int64_t lo(int c) const { int64_t v = piece * c; return v < n ? v : n; }
    int64_t hi(int c) const { int64_t v = piece * (c + 1); return v < n ? v : n; }
};

template <class E>
using Buf = std::vector<typename E::T>;

template <class E>
const typename E::T* in_ptr(const void* const* in, int p) {
    return static_cast<const typename E::T*>(in[p]);
}

template <class E>
typename E::T* out_ptr(void* const* out, int p) {
    return static_cast<typename E::T*>(out[p]);
}

/* Ascending-rank fp32 sum of element i over ranks first..first+count-1,
 * rounded once to the tensor type. */
template <class E>
typename E::T reduce_ranks(const void* const* in, int first, int count, int64_t i) {
    float acc = E::widen(in_ptr<E>(in, first)[i]);
    for (int q = first + 1; q < first + count; ++q) acc = add32(acc, E::widen(in_ptr<E>(in, q)[i]));
    return E::narrow(acc);
}

/* Same sum, kept in fp32 (no rounding): the fp32-wire variants. */
template <class E>
float reduce_ranks_f32(const void* const* in, int first, int count, int64_t i) {
    float acc = E::widen(in_ptr<E>(in, first)[i]);
    for (int q = first + 1; q < first + count; ++q) acc = add32(acc, E::widen(in_ptr<E>(in, q)[i]));
    return acc;
}

/* One-shot [CAR]: every rank reads all P inputs and reduces the whole vector
 * into its own output. */
template <class E>
void oneshot(const void* const* in, void* const* out, int P, int64_t n) {
    for (int r = 0; r < P; ++r)
        for (int64_t i = 0; i < n; ++i) out_ptr<E>(out, r)[i] = reduce_ranks<E>(in, 0, P, i);
}

/* 2-stage [CAR]. Stage 1 (reduce-scatter): rank c reduces the slice it owns
 * over all P inputs and stores it in its own output. Stage 2 (all-gather):
 * pull mode - rank r copies slice c out of rank c's output, for every c != r;
 * write mode - the owner stores its reduced slice straight into every rank's
 * output. */
template <class E>
void twostage(const void* const* in, void* const* out, int P, int64_t n, bool write_mode) {
    Split s(n, P, E::bytes);
    for (int c = 0; c < P; ++c) {
        for (int64_t i = s.lo(c); i < s.hi(c); ++i) {
            typename E::T v = reduce_ranks<E>(in, 0, P, i);
            if (write_mode) {
                for (int r = 0; r < P; ++r) out_ptr<E>(out, r)[i] = v;
            } else {
                out_ptr<E>(out, c)[i] = v;
            }
        }
    }
    if (write_mode) return;
    for (int r = 0; r < P; ++r)
        for (int c = 0; c < P; ++c) {
            if (c == r) continue;
            for (int64_t i = s.lo(c); i < s.hi(c); ++i) out_ptr<E>(out, r)[i] = out_ptr<E>(out, c)[i];
        }
}

/* Recursive doubling over `ranks` buffers (a power of two) on elements
 * [lo, hi), in place [NVRAR phase 2]. At step k rank p exchanges its current
 * partial with partner p XOR 2^k and keeps own + partner, rounded to the
 * tensor type. Each step reads only the values of the step before. The data
 * is processed in `chunks` contiguous chunks; a chunk's steps never touch
 * another chunk, so the chunk count changes scheduling, not values. */
template <class E>
void recursive_doubling(std::vector<Buf<E>>& v, int64_t lo, int64_t hi, int chunks) {
    const int ranks = static_cast<int>(v.size());
    if (chunks < 1) chunks = 1;
    const int64_t len = hi - lo;
    const int64_t V = 16 / E::bytes;
    const int64_t per = ((len + chunks - 1) / chunks + V - 1) / V * V;
    std::vector<Buf<E>> next(ranks, Buf<E>(v.empty() ? 0 : v[0].size()));
    for (int ch = 0; ch < chunks; ++ch) {
        int64_t a = lo + per * ch, b = a + per;
        if (a > hi) a = hi;
        if (b > hi) b = hi;
        for (int dist = 1; dist < ranks; dist <<= 1) {
            for (int p = 0; p < ranks; ++p) {
                const int q = p ^ dist;
                for (int64_t i = a; i < b; ++i)
                    next[p][i] = E::narrow(add32(E::widen(v[p][i]), E::widen(v[q][i])));
            }
            for (int p = 0; p < ranks; ++p)
                for (int64_t i = a; i < b; ++i) v[p][i] = next[p][i];
        }
    }
}

/* Flat recursive doubling all-reduce [NVRAR phase 2 applied to all P ranks]. */
template <class E>
void rd_allreduce(const void* const* in, void* const* out, int P, int64_t n, int chunks) {
    std::vector<Buf<E>> v(P, Buf<E>(n));
    for (int p = 0; p < P; ++p)
        for (int64_t i = 0; i < n; ++i) v[p][i] = in_ptr<E>(in, p)[i];
    recursive_doubling<E>(v, 0, n, chunks);
    for (int p = 0; p < P; ++p)
        for (int64_t i = 0; i < n; ++i) out_ptr<E>(out, p)[i] = v[p][i];
}

/* Flat recursive doubling with fp32 partials on the wire: the partials are
 * widened once, every step adds in fp32 without rounding (the same exchange
 * as above on fp32 buffers), and each rank rounds its result once at the end. */
template <class E>
void rd_allreduce_fp32wire(const void* const* in, void* const* out, int P, int64_t n, int chunks) {
    std::vector<Buf<F32>> v(P, Buf<F32>(n));
    for (int p = 0; p < P; ++p)
        for (int64_t i = 0; i < n; ++i) v[p][i] = E::widen(in_ptr<E>(in, p)[i]);
    recursive_doubling<F32>(v, 0, n, chunks);
    for (int p = 0; p < P; ++p)
        for (int64_t i = 0; i < n; ++i) out_ptr<E>(out, p)[i] = E::narrow(v[p][i]);
}

/* Hierarchical all-reduce with fp32 partials: the in-group sum is kept in
 * fp32, recursive doubling across groups adds in fp32, and the all-gather
 * stores the one rounding to the tensor type. */
template <class E>
void hier_allreduce_fp32wire(const void* const* in, void* const* out, int P, int64_t n, int L, int chunks) {
    const int G = P / L;
    Split s(n, L, E::bytes);
    std::vector<Buf<F32>> part(P, Buf<F32>(n));
    for (int g = 0; g < G; ++g)
        for (int l = 0; l < L; ++l)
            for (int64_t i = s.lo(l); i < s.hi(l); ++i) part[g * L + l][i] = reduce_ranks_f32<E>(in, g * L, L, i);
    for (int l = 0; l < L; ++l) {
        std::vector<Buf<F32>> across(G);
        for (int g = 0; g < G; ++g) across[g].swap(part[g * L + l]);
        recursive_doubling<F32>(across, s.lo(l), s.hi(l), chunks);
        for (int g = 0; g < G; ++g) across[g].swap(part[g * L + l]);
    }
    for (int g = 0; g < G; ++g)
        for (int l = 0; l < L; ++l)
            for (int lp = 0; lp < L; ++lp)
                for (int64_t i = s.lo(l); i < s.hi(l); ++i)
                    out_ptr<E>(out, g * L + lp)[i] = E::narrow(part[g * L + l][i]);
}

/* Hierarchical all-reduce [NVRAR]: P = G * L ranks in G groups of L, rank
 * r = g * L + l (group-major). Phase 1: in-group reduce-scatter - rank (g, l)
 * reduces slice l over the L ranks of group g in ascending order, one rounding.
 * Phase 2: for each slice l, recursive doubling across the G groups among the
 * ranks (0, l), (1, l), ..., (G-1, l). Phase 3: in-group all-gather - rank
 * (g, l) stores its slice into the outputs of all L ranks of its group. */
template <class E>
void hier_allreduce(const void* const* in, void* const* out, int P, int64_t n, int L, int chunks) {
    const int G = P / L;
    Split s(n, L, E::bytes);
    std::vector<Buf<E>> part(P, Buf<E>(n));  // part[r] holds rank r's slice only
    for (int g = 0; g < G; ++g)
        for (int l = 0; l < L; ++l)
            for (int64_t i = s.lo(l); i < s.hi(l); ++i) part[g * L + l][i] = reduce_ranks<E>(in, g * L, L, i);
    for (int l = 0; l < L; ++l) {
        std::vector<Buf<E>> across(G);
        for (int g = 0; g < G; ++g) across[g].swap(part[g * L + l]);
        recursive_doubling<E>(across, s.lo(l), s.hi(l), chunks);
        for (int g = 0; g < G; ++g) across[g].swap(part[g * L + l]);
    }
    for (int g = 0; g < G; ++g)
        for (int l = 0; l < L; ++l)
            for (int lp = 0; lp < L; ++lp)
                for (int64_t i = s.lo(l); i < s.hi(l); ++i) out_ptr<E>(out, g * L + lp)[i] = part[g * L + l][i];
}

/* Standalone reduce-scatter [NVRAR phase 1, all P ranks in one group]:
 * out[p] (n/P elements) is slice p of the ascending-rank sum. */
template <class E>
void reduce_scatter(const void* const* in, void* const* out, int P, int64_t n) {
    const int64_t m = n / P;
    for (int p = 0; p < P; ++p)
        for (int64_t j = 0; j < m; ++j) out_ptr<E>(out, p)[j] = reduce_ranks<E>(in, 0, P, p * m + j);
}

/* Standalone all-gather [NVRAR phase 3]: out[p] = in[0] | in[1] | ... | in[P-1]. */
template <class E>
void all_gather(const void* const* in, void* const* out, int P, int64_t n) {
    const int64_t m = n / P;
    for (int p = 0; p < P; ++p)
        for (int c = 0; c < P; ++c)
            for (int64_t j = 0; j < m; ++j) out_ptr<E>(out, p)[c * m + j] = in_ptr<E>(in, c)[j];
}


/* ---- OCP FP8 E4M3 and the fp8 wire (readings of ca_fp8_quant) ----------------- */

/* Round a binary32 to the nearest E4M3 value, ties to even, magnitudes past the
 * largest finite value (448) saturating to it. Values are kept as binary32
 * (every E4M3 value is exact in binary32). In the binade [2^e, 2^(e+1)) with
 * e >= -6 the E4M3 values are spaced 2^(e-3) apart; below 2^-6 (subnormals)
 * they are spaced 2^-9 apart. So the value is round_half_even(|v| / ulp) * ulp
 * with that spacing; both scalings are by powers of two and exact, and the
 * integer rounding is exact in binary32. */
inline float e4m3_round(float v) {
    const float a = v < 0.0f ? -v : v;
    if (!(a == a)) return v;  /* NaN stays NaN (inputs are finite in every use) */
    float ulp;
    if (a < 0.015625f) {      /* below 2^-6: subnormal spacing */
        ulp = 0.001953125f;   /* 2^-9 */
    } else {
        int e = 0;
        float m = a;
        while (m >= 2.0f) { m *= 0.5f; ++e; }
        while (m < 1.0f) { m *= 2.0f; --e; }
        ulp = 1.0f;
        for (int k = 0; k < e - 3; ++k) ulp *= 2.0f;
        for (int k = 0; k > e - 3; --k) ulp *= 0.5f;
    }
    const float t = a / ulp;                 /* exact: power-of-two scaling */
    float r = static_cast<float>(static_cast<int64_t>(t));   /* floor, t >= 0 */
    const float frac = t - r;                /* exact */
    if (frac > 0.5f || (frac == 0.5f && std::fmod(r, 2.0f) != 0.0f)) r += 1.0f;
    float q = r * ulp;                       /* exact */
    if (q > 448.0f) q = 448.0f;              /* saturate (RNE may step to 480 or beyond) */
    return v < 0.0f || (v == 0.0f && std::signbit(v)) ? -q : q;
}

/* Quantise and dequantise one group of `len` binary32 values in place. */
inline void fp8_group_qdq(float* x, int len) {
    float amax = 0.0f;
    for (int i = 0; i < len; ++i) {
        const float a = x[i] < 0.0f ? -x[i] : x[i];
        if (a > amax) amax = a;
    }
    volatile float s = amax / 448.0f;
    float sc = s;
    if (sc == 0.0f) sc = 1.0f;
    for (int i = 0; i < len; ++i) {
        volatile float t = x[i] / sc;
        volatile float d = e4m3_round(t) * sc;
        x[i] = d;
    }
}

/* Apply the fp8 wire to a whole vector of binary32 values: groups of 8. */
inline void fp8_wire(std::vector<float>& v) {
    const int64_t n = static_cast<int64_t>(v.size());
    for (int64_t g = 0; g < n; g += 8) fp8_group_qdq(v.data() + g, static_cast<int>(n - g < 8 ? n - g : 8));
}

/* Rank p's input as binary32 after the fp8 wire. */
template <class E>
std::vector<float> fp8_input(const void* const* in, int p, int64_t n) {
    std::vector<float> v(static_cast<size_t>(n));
    for (int64_t i = 0; i < n; ++i) v[i] = E::widen(in_ptr<E>(in, p)[i]);
    fp8_wire(v);
    return v;
}

/* One-shot with fp8 payloads: every rank reads all P inputs through the fp8
 * wire, adds them in ascending rank order in binary32, rounds once. */
template <class E>
void oneshot_fp8(const void* const* in, void* const* out, int P, int64_t n) {
    std::vector<std::vector<float>> x(P);
    for (int p = 0; p < P; ++p) x[p] = fp8_input<E>(in, p, n);
    for (int r = 0; r < P; ++r)
        for (int64_t i = 0; i < n; ++i) {
            float acc = x[0][i];
            for (int p = 1; p < P; ++p) acc = add32(acc, x[p][i]);
            out_ptr<E>(out, r)[i] = E::narrow(acc);
        }
}

/* 2-stage with fp8 payloads. Reduce-scatter: the owner of each slice adds
 * the P inputs, each through the fp8 wire, in ascending rank order in
 * binary32. All-gather: the reduced binary32 slice passes the fp8 wire again
 * (groups of 8 of the vector, which never straddle two slices: slices are
 * whole 16-byte items), and every rank stores it rounded to the tensor type.
 * Pull and write modes store the same values. */
template <class E>
void twostage_fp8(const void* const* in, void* const* out, int P, int64_t n) {
    Split sp(n, P, E::bytes);
    std::vector<std::vector<float>> x(P);
    for (int p = 0; p < P; ++p) x[p] = fp8_input<E>(in, p, n);
    std::vector<float> sum(static_cast<size_t>(n));
    for (int c = 0; c < P; ++c)
        for (int64_t i = sp.lo(c); i < sp.hi(c); ++i) {
            float acc = x[0][i];
            for (int p = 1; p < P; ++p) acc = add32(acc, x[p][i]);
            sum[i] = acc;
        }
    fp8_wire(sum);
    for (int r = 0; r < P; ++r)
        for (int64_t i = 0; i < n; ++i) out_ptr<E>(out, r)[i] = E::narrow(sum[i]);
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

enum Dt { DT_BF16 = 0, DT_F16 = 1, DT_F32 = 2 };

int dtype_code(const char* dt) {
    if (!dt) return -1;
    if (std::strcmp(dt, "bf16") == 0) return DT_BF16;
    if (std::strcmp(dt, "fp16") == 0) return DT_F16;
    if (std::strcmp(dt, "fp32") == 0) return DT_F32;
    return -1;
}

/* Element value of buffer x at index i as double (exact for all three types). */
double elem_as_double(const void* x, int64_t i, int dt) {
    if (dt == DT_BF16) return static_cast<double>(bf16_widen(static_cast<const uint16_t*>(x)[i]));
    if (dt == DT_F16) return static_cast<double>(half_widen(static_cast<const uint16_t*>(x)[i]));
    return static_cast<double>(static_cast<const float*>(x)[i]);
}

template <class E>
int allreduce_t(const char* algo, const void* const* in, void* const* out, int P, int64_t n, int L, int chunks) {
    if (std::strcmp(algo, "oneshot") == 0) { oneshot<E>(in, out, P, n); return 0; }
    if (std::strcmp(algo, "twostage") == 0) { twostage<E>(in, out, P, n, false); return 0; }
    if (std::strcmp(algo, "twostage_write") == 0) { twostage<E>(in, out, P, n, true); return 0; }
    if (std::strcmp(algo, "rd") == 0) {
        if (!is_pow2(P)) return -2;
        rd_allreduce<E>(in, out, P, n, chunks);
        return 0;
    }
    if (std::strcmp(algo, "hier") == 0) {
        if (L < 1 || P % L != 0 || !is_pow2(P / L)) return -2;
        hier_allreduce<E>(in, out, P, n, L, chunks);
        return 0;
    }
    if (std::strcmp(algo, "rd_fp32wire") == 0) {
        if (!is_pow2(P)) return -2;
        rd_allreduce_fp32wire<E>(in, out, P, n, chunks);
        return 0;
    }
    if (std::strcmp(algo, "hier_fp32wire") == 0) {
        if (L < 1 || P % L != 0 || !is_pow2(P / L)) return -2;
        hier_allreduce_fp32wire<E>(in, out, P, n, L, chunks);
        return 0;
    }
    const bool fp8 = std::strcmp(algo, "oneshot_fp8") == 0 || std::strcmp(algo, "twostage_fp8") == 0 ||
                     std::strcmp(algo, "twostage_write_fp8") == 0;
    if (fp8 && E::bytes != 2) return -2;  /* fp8 payloads are defined for 16-bit tensors */
    if (std::strcmp(algo, "oneshot_fp8") == 0) { oneshot_fp8<E>(in, out, P, n); return 0; }
    if (fp8) { twostage_fp8<E>(in, out, P, n); return 0; }
    return -1;
}

}  // namespace

extern "C" {

/* Round n binary32 values to bf16 bit patterns. */
void oracle_bf16_round(const float* x, uint16_t* y, int64_t n) {
    IeeeScope env;
    for (int64_t i = 0; i < n; ++i) y[i] = bf16_round(x[i]);
}

/* Widen n bf16 bit patterns to binary32. */
void oracle_bf16_widen(const uint16_t* x, float* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = bf16_widen(x[i]);
}

/* Round n binary32 values to fp16 bit patterns. */
void oracle_fp16_round(const float* x, uint16_t* y, int64_t n) {
    IeeeScope env;
    for (int64_t i = 0; i < n; ++i) y[i] = half_round(x[i]);
}

/* Widen n fp16 bit patterns to binary32. */
void oracle_fp16_widen(const uint16_t* x, float* y, int64_t n) {
    IeeeScope env;
    for (int64_t i = 0; i < n; ++i) y[i] = half_widen(x[i]);
}

/* Round n binary32 values to E4M3 values (returned as binary32). */
void oracle_e4m3_round(const float* x, float* y, int64_t n) {
    IeeeScope env;
    for (int64_t i = 0; i < n; ++i) y[i] = e4m3_round(x[i]);
}

/* The fp8 wire on n binary32 values (groups of 8 from index 0), in place. */
void oracle_fp8_wire(float* x, int64_t n) {
    IeeeScope env;
    std::vector<float> v(x, x + n);
    fp8_wire(v);
    for (int64_t i = 0; i < n; ++i) x[i] = v[i];
}

/* All-reduce of P rank buffers of n elements. algo: "oneshot", "twostage",
 * "twostage_write", "rd", "hier", "rd_fp32wire", "hier_fp32wire", "oneshot_fp8", "twostage_fp8",
 * "twostage_write_fp8" (the last three for bf16 / fp16 only); dtype: "bf16" or "fp16" (uint16 bit
 * patterns) or "fp32". L is the group size for "hier"; chunks is the chunk
 * count of the recursive-doubling phase. Returns 0, -1 (bad argument) or -2 (P/L shape the
 * algorithm does not define). */
int oracle_allreduce(const char* algo, const void* const* in, void* const* out, int P, int64_t n,
                     const char* dtype, int L, int chunks) {
    IeeeScope env;
    const int dt = dtype_code(dtype);
    if (!algo || !in || !out || P < 1 || n < 0 || dt < 0) return -1;
    if (n == 0) return 0;
    if (dt == DT_BF16) return allreduce_t<Bf16>(algo, in, out, P, n, L, chunks);
    if (dt == DT_F16) return allreduce_t<F16>(algo, in, out, P, n, L, chunks);
    return allreduce_t<F32>(algo, in, out, P, n, L, chunks);
}

/* Reduce-scatter: in[p] has n elements, out[p] has n / P; n % P == 0. */
int oracle_reduce_scatter(const void* const* in, void* const* out, int P, int64_t n, const char* dtype) {
    IeeeScope env;
    const int dt = dtype_code(dtype);
    if (!in || !out || P < 1 || n < 0 || dt < 0 || n % P != 0) return -1;
    if (dt == DT_BF16) reduce_scatter<Bf16>(in, out, P, n);
    else if (dt == DT_F16) reduce_scatter<F16>(in, out, P, n);
    else reduce_scatter<F32>(in, out, P, n);
    return 0;
}

/* All-gather: in[p] has n / P elements, out[p] has n; n % P == 0. */
int oracle_all_gather(const void* const* in, void* const* out, int P, int64_t n, const char* dtype) {
    const int dt = dtype_code(dtype);
    if (!in || !out || P < 1 || n < 0 || dt < 0 || n % P != 0) return -1;
    if (dt == DT_BF16) all_gather<Bf16>(in, out, P, n);
    else if (dt == DT_F16) all_gather<F16>(in, out, P, n);
    else all_gather<F32>(in, out, P, n);
    return 0;
}

/* fp64 reference: S[i] = sum over p of x_p[i] in double (ascending rank), and
 * the scale A[i] = sum over p of |x_p[i]|, which bounds every rounding error of
 * an fp32 or bf16 summation of the same terms. */
int oracle_fp64_reference(const void* const* in, int P, int64_t n, const char* dtype, double* S, double* A) {
    IeeeScope env;
    const int dt = dtype_code(dtype);
    if (!in || P < 1 || n < 0 || dt < 0 || !S || !A) return -1;
    for (int64_t i = 0; i < n; ++i) {
        double s = 0.0, a = 0.0;
        for (int p = 0; p < P; ++p) {
            const double x = elem_as_double(in[p], i, dt);
            s += x;
            a += x < 0 ? -x : x;
        }
        S[i] = s;
        A[i] = a;
    }
    return 0;
}

}  // extern "C"
