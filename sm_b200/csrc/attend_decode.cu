// Tuned decode attention: D = 128, 4- or 8-bit codes, groups of 32 or 8,
// four query heads per KV head (GQA), one query row per sequence.
//
// What it computes is the block rule of "Block KV decoding: less workspace,
// more time" (huhohoo.com/en/docs/llm/kv-block-decode-cost, section "Do not
// average independently normalized blocks") over the packed format of
// "KV分组打包：4-bit到底省了多少？" (huhohoo.com/docs/llm/kv-packed-groups,
// section "一个字节里到底装了什么"); each GQA group of four query heads reads its
// KV head once ("给长前缀列一张有单位的资源账本", section "GQA改变共享接口").
//
// Layout of the work
// ------------------
// * The concatenated (b, h, 32-token block) list is split evenly over
//   workers, one worker per warp pair (CTAs x pairs per CTA), each with a
//   contiguous range; a 32-token block is exactly one K group at g32 (one K
//   scale row serves the whole block) and four at g8 (each of the four lane
//   groups of a warp takes one).  After the prologue no barrier spans more
//   than a pair: every pair runs at its own pace.
// * Each pair runs one pipeline of bulk copies (cp.async.bulk, completion
//   counted on an mbarrier) carrying, per block, 32 tokens of K codes and V
//   codes, the block's K scale row(s) (512 B at g32, 2 KB at g8) and the
//   tokens' V scales (512 B at g32, 2 KB at g8).
//   - The S-warp (scores) keeps the segment's q in shared memory, folds the
//     K scales into it once per block, unpacks K once for all four heads and
//     writes per-lane partial scores; it also refills the pipeline.
//   - The V-warp (values) sums the partials into scores, runs the online
//     softmax (m, z) in log2 units (q carries scale * log2(e), so exp is one
//     ex2), rescales its accumulators when m grows and adds p * s_v * v for
//     its 16 channels and four heads with packed f32x2 FMAs.
//   Splitting the roles keeps each warp at 128 registers.
// * At the end of each (b, h) segment of its range the V-warp writes the
//   pair's state: the output if the range covered the segment whole, else a
//   partial (m, z, u) for the split merge kernel.
//
// Unpacking without a subtract
// ----------------------------
// A nibble n in mantissa bits [p, p+4) under exponent 0 reads as the float
// 1 + n * 2^(p-23).  Shifting a code word left by 15, 7 or right by 1, 9 puts
// the two nibbles of one byte at p = 15 and p = 19, so one LOP3 per code gives
// f = 1 + n * eps with eps = 2^-8 for even channels and 2^-4 for odd ones,
// and the two channels of a byte land in one f32x2 pair.  With q'' = q' / eps,
// sum q'' f - sum q'' (1 + 7 eps) = sum q' (n - 7): the second sum is one
// correction per block.  For V the subtraction is done per channel pair,
// f - (1 + 7 eps) = (n - 7) eps, which is exact, so u = sum p' (n - 7) eps
// carries no cancellation and a zero code contributes exactly zero.
#include "f32x2.cuh"
#include "kvq_internal.cuh"
#include "plan.cuh"
#include "quant.cuh"

namespace kvq {
namespace {

constexpr int kD = 128;
constexpr int kG = 4;                 // query heads per KV head
constexpr int kTB = 32;               // tokens per block (one K group)
// Per code width and group size: warp pairs per CTA, CTAs per SM, pipeline
// stages per pair, code bytes per token, scale layout.  4-bit g32: one CTA
// of eight pairs (three stages each) per SM, which measured a little faster
// than two CTAs of four: co-resident CTAs are not scheduled evenly, and the
// one the SM favours finishes well before the other.  8-bit g32 blocks
// carry twice the code bytes: three pairs of two stages, two CTAs per SM.
// g8 blocks carry four K scale rows and sixteen V scales per token: two
// stages, eight pairs (4-bit) or six (8-bit) in one CTA per SM.
template <int BITS, int GRP>
struct Tr {
  static_assert(GRP == 32 || GRP == 8, "group of 32 or 8 tokens / features");
  static constexpr int kNP = BITS == 4 ? 8 : (GRP == 32 ? 3 : 6);
  static constexpr int kCtasPerSm = (BITS == 8 && GRP == 32) ? 2 : 1;
  static constexpr int kS = (BITS == 4 && GRP == 32) ? 3 : 2;
  static constexpr int kThreads = 2 * kNP * 32;
  static constexpr int kCb = BITS == 4 ? 64 : 128;
  static constexpr int kKsRows = 32 / GRP;          // K scale rows (groups) per 32-token block
  static constexpr int kVs = 128 / GRP;             // V scales per token
  static constexpr int kPvW = GRP == 32 ? 20 : 4;   // floats per token row of the p table
  // How the pipeline refills.  Split: the S-warp streams each stage's K half
  // and the V-warp its V half, each refilling right after its own last read
  // (8-bit 114 -> 109 us, g8 slightly faster).  Whole: the S-warp refills
  // the whole stage once the V-warp has released it, which measured faster
  // at 4-bit g32 (91.8 us against 94.7 or 100.9 us split), where the
  // 128-register budget leaves no room for a second copy cursor.
  static constexpr bool kSplit = !(BITS == 4 && GRP == 32);
  // each channel's code f = 1 + code * eps sits in mantissa bits 15.. (even
  // 4-bit channels, every 8-bit channel: eps = 2^-8) or 19.. (odd 4-bit
  // channels: eps = 2^-4); corr = 1 + qmax * eps
  static constexpr float kInvEpsEven = 256.f;
  static constexpr float kInvEpsOdd = BITS == 4 ? 16.f : 256.f;
  static constexpr float kCorrEven = BITS == 4 ? 1.f + 7.f / 256.f : 1.f + 127.f / 256.f;
  static constexpr float kCorrOdd = BITS == 4 ? 1.f + 7.f / 16.f : 1.f + 127.f / 256.f;
};
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.f;          // rescale threshold of the running reference, log2 units
constexpr float kLn2 = 0.6931471805599453f;

template <int BITS, int GRP>
struct Stage {
  uint8_t kc[kTB * Tr<BITS, GRP>::kCb];    // K codes, 64 or 128 B per token
  uint8_t vc[kTB * Tr<BITS, GRP>::kCb];    // V codes
  float ks[Tr<BITS, GRP>::kKsRows][kD];    // K scale rows of the block's groups
  float vs[kTB][Tr<BITS, GRP>::kVs];       // V scales, 4 (g32) or 16 (g8) per token
};

template <int BITS, int GRP>
struct PairSmem {
  Stage<BITS, GRP> st[Tr<BITS, GRP>::kS];
  float qs[kG * kD];                  // q of the pair's current segment, * scale * log2e / eps,
                                      // swizzled (qs_index)
  float part[2][kTB * 32];            // score partials, double-buffered (part_index)
  float pv[kTB][Tr<BITS, GRP>::kPvW];  // g32: p' = p * s_v of token t, group g, head h at
                                      // [t][4g + h], four entries pad the row; g8: p of token
                                      // t, head h at [t][h] (the V scale goes on the codes)
  unsigned long long full[Tr<BITS, GRP>::kS];    // split: the K half landed; whole: the stage landed
  unsigned long long other[Tr<BITS, GRP>::kS];   // split: the V half landed; whole: the V-warp
                                                 // released the stage
  unsigned long long cursor[2][6];    // each warp's copy cursor (a Prod), lane 0's alone
  unsigned long long pfull[2];        // S-warp wrote part[i]
  unsigned long long pempty[2];       // V-warp read part[i]
  int abort;                          // a wait of this pair ran out: both warps stop
  unsigned int issued[2];             // copies each warp issued (lane 0 counts): drained on an abort
  int pad_;
};

static_assert(sizeof(Stage<4, 32>) % 16 == 0 && sizeof(Stage<8, 32>) % 16 == 0 &&
                  sizeof(Stage<4, 8>) % 16 == 0 && sizeof(Stage<8, 8>) % 16 == 0,
              "stage alignment");
static_assert(sizeof(PairSmem<4, 32>) % 16 == 0 && sizeof(PairSmem<8, 32>) % 16 == 0 &&
                  sizeof(PairSmem<4, 8>) % 16 == 0 && sizeof(PairSmem<8, 8>) % 16 == 0,
              "pair alignment");

struct DecodeParams {
  const void* Q;
  int q_dtype;
  const uint8_t* k_codes;
  const float* k_scales;
  const uint8_t* v_codes;
  const float* v_scales;
  const int32_t* lengths;
  int B, H, N_cap;
  long long k_codes_head, k_scales_head, v_codes_head, v_scales_head;
  float qscale;                       // scale * log2(e)
  void* O;
  float* partials;                    // [slots][kG][kD + 2]
  int ctas;                           // CTAs; each warp pair is one worker of the plan
  int force_partial;                  // a window follows: no worker writes output rows
  unsigned int* err;
  unsigned long long wait_ns;         // limit of every bounded wait
  int lose_worker, lose_block;        // self-test of the timeout path: this worker's K copy of its
                                      // lose_block-th block arms 16 bytes more than it brings, so
                                      // that block's barrier never completes; -1: none
  // decode step (kvq_decode_step): each sequence's new token t = lengths[b] - 1
  // is appended first -- its K group re-packed from k_tail [B, H, GRP, kD], V
  // row t from v_new [B, H, kD] -- by the worker that owns the (b, h)'s last
  // block; nullptr: no append
  const void* k_tail;
  const void* v_new;
  int in_dtype;
};

// shared memory after the pairs: pre [B + 1], len [B]
template <int BITS, int GRP>
size_t smem_bytes(int B) {
  return sizeof(PairSmem<BITS, GRP>) * Tr<BITS, GRP>::kNP + sizeof(int) * (2 * B + 1);
}

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(unsigned long long* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(unsigned long long* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete
// sleeps in hardware (up to the hint, in ns) instead of polling.
__device__ __forceinline__ bool mbar_try_wait_sleep(unsigned long long* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(200000u)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Orders this thread's earlier generic-proxy accesses of shared memory before
// its later async-proxy (bulk copy) writes to it.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on a phase of `bar`: true once the phase completed.  It gives
// up -- returns false -- when the pair's abort flag is up (the other warp gave
// up), or after limit_ns, when it raises the flag itself and records
// KVQ_ERR_TIMEOUT.  Callers go on either way (their next shared-memory reads
// may then see stale data, which is harmless); each warp checks the flag once
// per block and leaves its loop, so one lost completion ends the pair's work
// within one limit and every later wait returns at once.
__device__ __forceinline__ bool wait_bar(unsigned long long* bar, uint32_t parity, unsigned int* err,
                                         volatile int* abort, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if ((it & 7u) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > limit_ns) {
        *abort = 1;
        record_error(err, KVQ_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// After an abort: wait (at most about two seconds) for a bulk copy this warp
// issued into `bar` to land, so no copy is still writing shared memory when
// the CTA exits.
__device__ __forceinline__ void drain_bar(unsigned long long* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_sleep(bar, parity)) return;
    if ((it & 7u) == 0 && globaltimer() - t0 > 2000000000ull) return;
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// Channel pairs (16cs + 2i, 16cs + 2i + 1), i = 0..7, of one 64-bit code load.
__device__ __forceinline__ void nibble_pairs(uint32_t w0, uint32_t w1, u64 f[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w = i < 4 ? w0 : w1;
    const int r = i & 3;
    f[i] = nibble_pair(byte_at15(w, r));
  }
}

// Channel pairs (16cs + 2i, 16cs + 2i + 1), i = 0..7, of a 16-byte load of
// 8-bit codes: each byte shifted to mantissa bits 15..22 of 1.0, so
// f = 1 + c * 2^-8 for every channel.
__device__ __forceinline__ void byte_pairs15(const uint4& w4, u64 f[8]) {
  const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t x = w[i >> 1];
    const int r = 2 * (i & 1);
    const uint32_t a = r == 0 ? (x << 15) : (x >> 1);            // byte r at bits 15..22
    const uint32_t b = r == 0 ? (x << 7) : (x >> 9);             // byte r + 1
    u64 v;
    asm("{.reg .b32 t0, t1;\n\t"
        "lop3.b32 t0, %1, 0x007F8000, 0x3F800000, 0xEA;\n\t"
        "lop3.b32 t1, %2, 0x007F8000, 0x3F800000, 0xEA;\n\t"
        "mov.b64 %0, {t0, t1};}"
        : "=l"(v)
        : "r"(a), "r"(b));
    f[i] = v;
  }
}

// The 16 channels (8 pairs) of lane slice cs of token t from a stage's codes.
template <int BITS>
__device__ __forceinline__ void code_pairs(const uint8_t* codes, int t, int cs, u64 f[8]) {
  if (BITS == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(codes + t * 64 + cs * 8);
    nibble_pairs(w.x, w.y, f);
  } else {
    const uint4 w = *reinterpret_cast<const uint4*>(codes + t * 128 + cs * 16);
    byte_pairs15(w, f);
  }
}

// V codes as exact offsets (code - qmax) * eps with one shift per four
// bytes.  The offset is taken per pair as f - (1 + qmax eps), which is exact
// for any eps (both terms lie in [1, 2)), so V needs no cancellation-safe
// placement: a code may sit anywhere its mantissa field stays below the
// exponent.  Per 32-bit word w (channels in byte order) and v = w >> 16, the
// channels keep their order: 4-bit pairs (ch 0, ch 1) and (ch 4, ch 5) at
// eps (2^-23, 2^-19), from w and v; (ch 2, ch 3) and (ch 6, ch 7) at
// (2^-15, 2^-11).  8-bit pairs (ch 0, ch 1) and (ch 2, ch 3) at
// (2^-23, 2^-15).  So two correction pairs at 4 bits and one at 8.
template <int BITS>
struct VSlot {
  // 1/eps of half j of pair i, at [2i + j]
  static constexpr float inv_eps(int k) {
    return BITS == 4 ? ((k & 3) == 0 ? 8388608.f : (k & 3) == 1 ? 524288.f : (k & 3) == 2 ? 32768.f : 2048.f)
                     : ((k & 1) == 0 ? 8388608.f : 32768.f);
  }
};

__device__ __forceinline__ uint32_t mant_or(uint32_t x, uint32_t mask) {
  uint32_t y;
  asm("lop3.b32 %0, %1, %2, 0x3F800000, 0xEA;" : "=r"(y) : "r"(x), "r"(mask));
  return y;
}

__device__ __forceinline__ u64 pair_u32(uint32_t lo, uint32_t hi) {
  u64 v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(lo), "r"(hi));
  return v;
}

// 1 + qmax * 2^(p - 23)
constexpr float vcorr(int qmax, int p) { return 1.f + static_cast<float>(qmax) / static_cast<float>(1 << (23 - p)); }

// The lane's 16 V channels of token t as eight exact offset pairs, channel
// 2i and 2i + 1 in pair i.
template <int BITS>
__device__ __forceinline__ void v_offsets(const uint8_t* codes, int t, int cs, u64 f[8]) {
  if (BITS == 4) {
    const uint2 w2 = *reinterpret_cast<const uint2*>(codes + t * 64 + cs * 8);
    const u64 c01 = pack2(-vcorr(7, 0), -vcorr(7, 4)), c23 = pack2(-vcorr(7, 8), -vcorr(7, 12));
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint32_t w = (h < 2 ? w2.x : w2.y) >> (16 * (h & 1));
      f[2 * h] = add2(pair_u32(mant_or(w, 0x000Fu), mant_or(w, 0x00F0u)), c01);
      f[2 * h + 1] = add2(pair_u32(mant_or(w, 0x0F00u), mant_or(w, 0xF000u)), c23);
    }
  } else {
    const uint4 w4 = *reinterpret_cast<const uint4*>(codes + t * 128 + cs * 16);
    const uint32_t ws[4] = {w4.x, w4.y, w4.z, w4.w};
    const u64 c = pack2(-vcorr(127, 0), -vcorr(127, 8));
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const uint32_t w = ws[h >> 1] >> (16 * (h & 1));
      f[h] = add2(pair_u32(mant_or(w, 0x00FFu), mant_or(w, 0xFF00u)), c);
    }
  }
}

// q of the segment lives in shared memory pre-scaled by 1/eps, with the four
// 16-byte chunks of each lane's 16 channels rotated so the eight lanes of a
// quarter warp hit eight different bank groups.
__device__ __forceinline__ int qs_index(int h, int c) {
  const int cs = c >> 4, j = (c >> 2) & 3;
  return h * kD + cs * 16 + ((j ^ ((cs >> 1) & 3)) << 2) + (c & 3);
}

// Token of lane group ts at iteration it of a block.  g32: tokens 4 it + ts,
// all of one K group.  g8: lane group ts owns K group ts (tokens 8 ts ..
// 8 ts + 7), visited in a rotated order so that the four groups' code rows
// fall in both halves of the shared-memory banks.
template <int GRP>
__device__ __forceinline__ int block_token(int it, int ts) {
  return GRP == 32 ? 4 * it + ts : 8 * ts + ((it + ts) & 7);
}

// Score partials of token t: the eight channel slices' float4 (one value per
// head) in a 128-byte row, slice i at float4 (i ^ (t & 7)) so that eight
// lanes reading slice i of eight tokens hit eight different bank groups.
__device__ __forceinline__ int part_index(int t, int i) { return t * 32 + ((i ^ (t & 7)) << 2); }

// ---------------------------------------------------------------------------
// iteration over a worker's block range
// ---------------------------------------------------------------------------
// A segment is the part of one head that a worker's range covers: plan
// slots [jb, jb + span) of the head's nb, at global slot gpos, and its blocks
// [jb, je).  The blocks stop at the head's last block: the decode step's
// plan has one more slot per head (its append, warp_block_prefix's extra),
// which holds no block, so a segment can hold that slot alone (jb == je).
struct Seg {
  int b, h, nb, jb, je;
  long long gpos;                     // global index of slot jb
  bool valid;
};

// Blocks of a sequence of clamped length len.
__device__ __forceinline__ int real_blocks(int len) { return (len + kTB - 1) / kTB; }

// SLOT: the decode step's plan with the append slot; without it a head's
// slots are its blocks.
template <bool SLOT>
__device__ __forceinline__ int seg_blocks(const Seg& s, const int* slen) {
  return SLOT ? real_blocks(slen[s.b]) : s.nb;
}

template <bool SLOT>
__device__ __forceinline__ Seg first_seg(const int* pre, const int* slen, int B, int H, const CtaRange& cr) {
  Seg s;
  s.valid = cr.g0 < cr.g1;
  if (!s.valid) return s;
  s.b = find_seq(pre, B, H, cr.g0);
  s.nb = pre[s.b + 1] - pre[s.b];
  const long long off = cr.g0 - static_cast<long long>(H) * pre[s.b];
  s.h = static_cast<int>(off / s.nb);
  s.jb = static_cast<int>(off % s.nb);
  s.je = static_cast<int>(min(static_cast<long long>(seg_blocks<SLOT>(s, slen)), s.jb + (cr.g1 - cr.g0)));
  s.gpos = cr.g0;
  return s;
}

template <bool SLOT>
__device__ __forceinline__ Seg next_seg(Seg s, const int* pre, const int* slen, int B, int H, const CtaRange& cr) {
  // past the segment's slots (its blocks, and the append slot if it holds it)
  s.gpos += SLOT ? min(static_cast<long long>(s.nb), s.jb + (cr.g1 - s.gpos)) - s.jb : s.je - s.jb;
  if (s.gpos >= cr.g1) {
    s.valid = false;
    return s;
  }
  if (++s.h == H) {
    s.h = 0;
    ++s.b;
    while (s.b < B && pre[s.b + 1] == pre[s.b]) ++s.b;
  }
  s.nb = pre[s.b + 1] - pre[s.b];
  s.jb = 0;
  s.je = static_cast<int>(min(static_cast<long long>(seg_blocks<SLOT>(s, slen)), cr.g1 - s.gpos));
  return s;
}

struct Prod {
  Seg seg;
  int j;
  bool valid;
};

template <bool SLOT>
__device__ __forceinline__ Prod prod_settle(Prod p, const int* pre, const int* slen, int B, int H,
                                            const CtaRange& cr) {
  while (p.valid && p.j >= p.seg.je) {
    p.seg = next_seg<SLOT>(p.seg, pre, slen, B, H, cr);
    p.valid = p.seg.valid;
    p.j = p.seg.jb;
  }
  return p;
}

// Whole refill: lane 0 arms the stage's barrier with the block's byte count
// and issues the four copies: K codes, V codes, the K scale rows of the
// block's groups holding valid tokens, and the V scales.
template <int BITS, int GRP>
__device__ __forceinline__ void issue_block(const DecodeParams& p, PairSmem<BITS, GRP>& ps, int stage, int b,
                                            int h, int j, const int* slen, uint32_t extra) {
  const long long head = static_cast<long long>(b) * p.H + h;
  const int len = slen[b];
  const int t0 = j * kTB;
  const int nv = min(kTB, len - t0);
  constexpr int kCb = Tr<BITS, GRP>::kCb;
  Stage<BITS, GRP>& st = ps.st[stage];
  unsigned long long* bar = &ps.full[stage];
  constexpr int kVs = Tr<BITS, GRP>::kVs;
  const int krows = (nv + GRP - 1) / GRP;                // K groups holding valid tokens
  mbar_expect_tx(bar, static_cast<uint32_t>((2 * kCb + kVs * 4) * nv + krows * kD * 4) + extra);
  bulk_g2s(st.kc, p.k_codes + head * p.k_codes_head + static_cast<long long>(t0) * kCb, nv * kCb, bar);
  bulk_g2s(st.vc, p.v_codes + head * p.v_codes_head + static_cast<long long>(t0) * kCb, nv * kCb, bar);
  bulk_g2s(st.ks, p.k_scales + head * p.k_scales_head + static_cast<long long>(t0 / GRP) * kD,
           krows * kD * sizeof(float), bar);
  bulk_g2s(st.vs, p.v_scales + head * p.v_scales_head + static_cast<long long>(t0) * kVs,
           nv * kVs * 4, bar);
}

// Split refill: the S-warp streams the K half of each stage (K codes, the K
// scale rows of the block's groups holding valid tokens) and the V-warp the
// V half (V codes, V scales): each warp is the only reader of its half, so
// it refills a stage as soon as its own reads of it are done.  Lane 0 arms
// the half's barrier with its byte count and issues its two copies.
template <int BITS, int GRP>
__device__ __forceinline__ void issue_half(const DecodeParams& p, PairSmem<BITS, GRP>& ps, int stage, int b,
                                           int h, int j, const int* slen, bool k_half, uint32_t extra) {
  const long long head = static_cast<long long>(b) * p.H + h;
  const int len = slen[b];
  const int t0 = j * kTB;
  const int nv = min(kTB, len - t0);
  constexpr int kCb = Tr<BITS, GRP>::kCb;
  constexpr int kVs = Tr<BITS, GRP>::kVs;
  Stage<BITS, GRP>& st = ps.st[stage];
  if (k_half) {
    unsigned long long* bar = &ps.full[stage];
    const int krows = (nv + GRP - 1) / GRP;                // K groups holding valid tokens
    mbar_expect_tx(bar, static_cast<uint32_t>(kCb * nv + krows * kD * 4) + extra);
    bulk_g2s(st.kc, p.k_codes + head * p.k_codes_head + static_cast<long long>(t0) * kCb, nv * kCb, bar);
    bulk_g2s(st.ks, p.k_scales + head * p.k_scales_head + static_cast<long long>(t0 / GRP) * kD,
             krows * kD * sizeof(float), bar);
  } else {
    unsigned long long* bar = &ps.other[stage];
    mbar_expect_tx(bar, static_cast<uint32_t>((kCb + kVs * 4) * nv));
    bulk_g2s(st.vc, p.v_codes + head * p.v_codes_head + static_cast<long long>(t0) * kCb, nv * kCb, bar);
    bulk_g2s(st.vs, p.v_scales + head * p.v_scales_head + static_cast<long long>(t0) * kVs, nv * kVs * 4, bar);
  }
}

// The decode step's append for one (b, h), by the 64 threads of a pair (pt =
// 0..63 handles channels 2 pt, 2 pt + 1): re-pack K group t / GRP of the new
// token t from the caller's float rows of that group (rows past t % GRP read
// as zero, as a whole-cache pack pads a short last group) and pack V row t,
// into the cache, with the arithmetic of the pack kernels, so the bytes are
// those a whole-cache pack of tokens [0, t] writes.
template <int BITS, int GRP>
__device__ __forceinline__ void append_tail(const DecodeParams& p, int b, int h, int t, int pt) {
  constexpr int qmax = BITS == 4 ? 7 : 127;
  const long long head = static_cast<long long>(b) * p.H + h;
  const int j = t / GRP, nin = t % GRP + 1;
  const int c = 2 * pt;
  // the group's rows of channels c, c + 1; the dtype branch sits outside the
  // row loop so the 2 GRP loads go out back to back (one round trip).  At 4
  // bits the new V row's two channels go out in the same batch: the worker
  // that appends covers one block fewer (the plan's append slot), which
  // leaves it off the tail only if the append costs one round trip (at 8
  // bits, without the slot, the batched form measured slower)
  float x0[GRP], x1[GRP], v0 = 0.f, v1 = 0.f;
  const long long e0 = head * GRP * kD + c;
  const long long ve = head * kD + c;
  if (p.in_dtype == KVQ_F32) {
    const float* src = static_cast<const float*>(p.k_tail) + e0;
#pragma unroll
    for (int r = 0; r < GRP; ++r) {
      x0[r] = r < nin ? src[r * kD] : 0.f;
      x1[r] = r < nin ? src[r * kD + 1] : 0.f;
    }
    if (BITS == 4) {
      v0 = static_cast<const float*>(p.v_new)[ve];
      v1 = static_cast<const float*>(p.v_new)[ve + 1];
    }
  } else {
    const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(p.k_tail) + e0;
#pragma unroll
    for (int r = 0; r < GRP; ++r) {
      x0[r] = r < nin ? __bfloat162float(src[r * kD]) : 0.f;
      x1[r] = r < nin ? __bfloat162float(src[r * kD + 1]) : 0.f;
    }
    if (BITS == 4) {
      v0 = __bfloat162float(static_cast<const __nv_bfloat16*>(p.v_new)[ve]);
      v1 = __bfloat162float(static_cast<const __nv_bfloat16*>(p.v_new)[ve + 1]);
    }
  }
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int r = 0; r < GRP; ++r) {
    a0 = fmaxf(a0, fabsf(x0[r]));
    a1 = fmaxf(a1, fabsf(x1[r]));
  }
  const float s0 = group_scale(a0, qmax), s1 = group_scale(a1, qmax);
  const float r0 = __frcp_rn(s0), r1 = __frcp_rn(s1);
  *reinterpret_cast<float2*>(const_cast<float*>(p.k_scales) + head * p.k_scales_head + static_cast<long long>(j) * kD +
                             c) = make_float2(s0, s1);
  uint8_t* kc = const_cast<uint8_t*>(p.k_codes) + head * p.k_codes_head;
#pragma unroll
  for (int r = 0; r < GRP; ++r) {
    const unsigned q0 = quant_code(x0[r], s0, r0, qmax), q1 = quant_code(x1[r], s1, r1, qmax);
    const long long row = static_cast<long long>(j) * GRP + r;
    if (BITS == 4) kc[row * 64 + pt] = static_cast<uint8_t>(q0 | (q1 << 4));
    else *reinterpret_cast<uint16_t*>(kc + row * 128 + c) = static_cast<uint16_t>(q0 | (q1 << 8));
  }
  // V row t: the GRP / 2 threads of a V group (within one warp) share its max
  if (BITS != 4) {
    v0 = load_as_f32(p.v_new, ve, p.in_dtype);
    v1 = load_as_f32(p.v_new, ve + 1, p.in_dtype);
  }
  float am = fmaxf(fabsf(v0), fabsf(v1));
#pragma unroll
  for (int o = 1; o < GRP / 2; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const float sv = group_scale(am, qmax), rv = __frcp_rn(sv);
  if ((c % GRP) == 0)
    const_cast<float*>(p.v_scales)[head * p.v_scales_head + static_cast<long long>(t) * (kD / GRP) + c / GRP] = sv;
  uint8_t* vc = const_cast<uint8_t*>(p.v_codes) + head * p.v_codes_head + static_cast<long long>(t) * (kD * BITS / 8);
  const unsigned w0 = quant_code(v0, sv, rv, qmax), w1 = quant_code(v1, sv, rv, qmax);
  if (BITS == 4) vc[pt] = static_cast<uint8_t>(w0 | (w1 << 4));
  else *reinterpret_cast<uint16_t*>(vc + c) = static_cast<uint16_t>(w0 | (w1 << 8));
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// APPEND: the decode step's form, which appends each sequence's new token
// first (a separate instantiation, so the plain attend carries none of it).
template <int BITS, int GRP, bool APPEND>
__global__ void __launch_bounds__(Tr<BITS, GRP>::kThreads, Tr<BITS, GRP>::kCtasPerSm) decode_kernel(DecodeParams p) {
  griddep_wait();
  // the append slot in the plan (Seg): 4-bit codes only, whose 1,184 workers
  // leave the split room for it at the decode workload's size (32,768 blocks
  // and 256 slots in ranges of 28).  Where there is no room (8-bit: 888
  // workers, ranges of 37 that the slots would make 38) every range grows by
  // one slot, so 8-bit keeps the plain plan; a runtime choice between the two
  // measured slower than either at 4 bits.
  constexpr bool kSlot = APPEND && BITS == 4;
  constexpr int kNP = Tr<BITS, GRP>::kNP, kS = Tr<BITS, GRP>::kS, kThreads = Tr<BITS, GRP>::kThreads;
  using PairSmem = kvq::PairSmem<BITS, GRP>;
  using Stage = kvq::Stage<BITS, GRP>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  PairSmem* pairs = reinterpret_cast<PairSmem*>(smem_raw);
  int* pre = reinterpret_cast<int*>(pairs + kNP);       // [B + 1]
  int* slen = pre + p.B + 1;                             // [B] lengths clamped to [0, N_cap]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool is_s = warp < kNP;                          // S-warp (scores) or V-warp (values)
  const int pair = is_s ? warp : warp - kNP;
  const int ts = lane >> 3, cs = lane & 7;
  PairSmem& ps = pairs[pair];

  // the decode step counts its append as one more plan slot per head (Seg):
  // the workers that append cover one block fewer
  if (warp == 0) warp_block_prefix(p.lengths, p.B, p.N_cap, kTB, pre, false, kSlot ? 1 : 0);
  for (int b = threadIdx.x; b < p.B; b += kThreads) slen[b] = clamp_len(p.lengths[b], p.N_cap);
  if (is_s && lane == 0) {
#pragma unroll
    for (int s = 0; s < kS; ++s) {
      mbar_init(&ps.full[s], 1);
      mbar_init(&ps.other[s], 1);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ps.pfull[i], 1);
      mbar_init(&ps.pempty[i], 1);
    }
    ps.abort = 0;
    ps.issued[0] = ps.issued[1] = 0;
  }
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncthreads();

  // From here on every warp pair works alone: it is worker blockIdx.x * kNP +
  // pair of the plan, with a contiguous block range of its own, and no
  // CTA-wide barrier follows.
  const int H = p.H;
  const int worker = blockIdx.x * kNP + pair;
  const CtaRange cr = cta_range(pre, p.B, H, p.ctas * kNP, worker);
  if (cr.g0 >= cr.g1) return;

  Seg seg = first_seg<kSlot>(pre, slen, p.B, H, cr);
  if (APPEND) {
    // decode step: append the new token of every (b, h) whose last block
    // this pair owns (only this pair reads that block), before any copy of
    // it is issued; the bulk copies read the cache through the async proxy
    for (Seg sg = seg; sg.valid; sg = next_seg<kSlot>(sg, pre, slen, p.B, H, cr)) {
      const int raw = p.lengths[sg.b];
      const bool last = kSlot ? (sg.jb < sg.je && sg.je == real_blocks(slen[sg.b])) : (sg.je == sg.nb);
      if (last && raw >= 1 && raw <= p.N_cap)
        append_tail<BITS, GRP>(p, sg.b, sg.h, raw - 1, (is_s ? 0 : 32) + lane);
    }
    asm volatile("fence.proxy.async;" ::: "memory");
    asm volatile("bar.sync %0, %1;" ::"r"(1 + pair), "r"(64) : "memory");
  }
  constexpr bool kSplit = Tr<BITS, GRP>::kSplit;
  // Whole refill: the S-warp's copy cursor, in registers.  Split refill:
  // each warp's cursor lives in shared memory and only lane 0 touches it, so
  // it takes no registers in the lanes' loops.
  Prod prod{seg, seg.jb, true};
  prod = prod_settle<kSlot>(prod, pre, slen, p.B, H, cr);
  static_assert(sizeof(Prod) <= sizeof(unsigned long long) * 6, "cursor slot");
  Prod* cur = reinterpret_cast<Prod*>(ps.cursor[is_s ? 0 : 1]);
  // S-warp: q of a segment, loaded (lane + 32 r) before it is scaled into qs.
  // The first segment's loads go out before the first block copies so they
  // do not queue behind them.
  constexpr int kPer = kG * kD / 32;
  float qv[kPer];
  auto load_q = [&](const Seg& sg) {
    const long long qrow = (static_cast<long long>(sg.b) * H + sg.h) * kG;
#pragma unroll
    for (int r = 0; r < kPer; ++r) qv[r] = load_as_f32(p.Q, qrow * kD + lane + 32 * r, p.q_dtype);
  };
  // q * scale * log2e / eps into the pair's qs (the channel of value r is
  // lane + 32 r, so its parity is the lane's)
  auto store_q = [&]() {
    const float qf = p.qscale * ((lane & 1) ? Tr<BITS, GRP>::kInvEpsOdd : Tr<BITS, GRP>::kInvEpsEven);
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int i = lane + 32 * r;
      ps.qs[qs_index(i / kD, i % kD)] = qv[r] * qf;
    }
  };
  // Copies this warp issued (whole refill: the S-warp's blocks; split: each
  // warp's halves), counted in shared memory by lane 0, the issuer: after an
  // abort the last kS of them are drained before the CTA exits.
  unsigned int* issued = &ps.issued[is_s ? 0 : 1];
  // the self-test's lost completion: 16 bytes armed that no copy brings
  auto extra_tx = [&](bool k_half) -> uint32_t {
    return (k_half && worker == p.lose_worker && *issued == static_cast<uint32_t>(p.lose_block)) ? 16u : 0u;
  };
  volatile int* abort = &ps.abort;
  if (is_s) load_q(seg);
  if constexpr (kSplit) {
    if (lane == 0) {
      Prod pr = prod;
      for (int s = 0; s < kS && pr.valid; ++s) {
        issue_half<BITS, GRP>(p, ps, s, pr.seg.b, pr.seg.h, pr.j, slen, is_s, extra_tx(is_s));
        ++*issued;
        ++pr.j;
        pr = prod_settle<kSlot>(pr, pre, slen, p.B, H, cr);
      }
      *cur = pr;
    }
  } else if (is_s) {
    for (int s = 0; s < kS && prod.valid; ++s) {
      if (lane == 0) {
        issue_block<BITS, GRP>(p, ps, s, prod.seg.b, prod.seg.h, prod.j, slen, extra_tx(true));
        ++*issued;
      }
      ++prod.j;
      prod = prod_settle<kSlot>(prod, pre, slen, p.B, H, cr);
    }
  }
  if (is_s) store_q();

  uint32_t k = 0;                                        // blocks this pair has consumed
  bool first = true;
  bool alive = true;                                     // no wait of the pair ran out
  while (seg.valid && alive) {
    const int b = seg.b, h = seg.h;
    const long long head = static_cast<long long>(b) * H + h;
    const long long qrow = static_cast<long long>(b) * H * kG + static_cast<long long>(h) * kG;
    const int len = slen[b];

    if (is_s) {
      // ===================== S-warp: partial scores =====================
      // the segment's q, pre-scaled by 1/eps; only this warp reads it
      float* qs = ps.qs;
      if (!first) {
        load_q(seg);
        store_q();
      }
      __syncwarp();
      for (int j = seg.jb; j < seg.je; ++j, ++k) {
        const int stage = static_cast<int>(k % kS);
        const int pb = static_cast<int>(k & 1u);
        if (*abort) {                                    // a wait of this pair ran out
          alive = false;
          break;
        }
        wait_bar(&ps.full[stage], (k / kS) & 1u, p.err, abort, p.wait_ns);
        const Stage& st = ps.st[stage];

        // q'' = q * scale * log2e / eps * s_k, as channel pairs (16cs + 2i, +1)
        u64 q2[kG][8];
        u64 kcp[kG];
        {
          // the K scales of this lane's group: the block's one group (g32) or
          // group ts (g8)
          const ulonglong2* ksv = reinterpret_cast<const ulonglong2*>(st.ks[GRP == 32 ? 0 : ts] + 16 * cs);
          ulonglong2 kv2[4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) kv2[jj] = ksv[jj];
          const u64 corr = pack2(Tr<BITS, GRP>::kCorrEven, Tr<BITS, GRP>::kCorrOdd);
#pragma unroll
          for (int hh = 0; hh < kG; ++hh) {
            u64 c2 = 0ull;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const ulonglong2 a2 = *reinterpret_cast<const ulonglong2*>(
                  qs + hh * kD + cs * 16 + ((jj ^ ((cs >> 1) & 3)) << 2));
              q2[hh][2 * jj] = mul2(a2.x, kv2[jj].x);
              q2[hh][2 * jj + 1] = mul2(a2.y, kv2[jj].y);
              c2 = fma2(q2[hh][2 * jj], corr, c2);
              c2 = fma2(q2[hh][2 * jj + 1], corr, c2);
            }
            kcp[hh] = static_cast<u64>(__float_as_uint(-(lo_f(c2) + hi_f(c2))));
          }
        }
        // the V-warp must have read this partial buffer's previous block
        if (k >= 2) wait_bar(&ps.pempty[pb], ((k - 2) >> 1) & 1u, p.err, abort, p.wait_ns);
        float* part = ps.part[pb];
#pragma unroll 2
        for (int it = 0; it < kTB / 4; ++it) {
          const int t = block_token<GRP>(it, ts);
          u64 f[8];
          code_pairs<BITS>(st.kc, t, cs, f);
          u64 acc[kG];
#pragma unroll
          for (int hh = 0; hh < kG; ++hh) {
            acc[hh] = fma2(q2[hh][0], f[0], kcp[hh]);
#pragma unroll
            for (int i = 1; i < 8; ++i) acc[hh] = fma2(q2[hh][i], f[i], acc[hh]);
          }
          *reinterpret_cast<float4*>(part + part_index(t, cs)) =
              make_float4(lo_f(acc[0]) + hi_f(acc[0]), lo_f(acc[1]) + hi_f(acc[1]),
                          lo_f(acc[2]) + hi_f(acc[2]), lo_f(acc[3]) + hi_f(acc[3]));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ps.pfull[pb]);

        if constexpr (kSplit) {
          // this warp has read the stage's K half for the last time: refill
          // it with the block kS ahead
          if (lane == 0) {
            Prod pr = *cur;
            if (pr.valid && !*abort) {                   // no new copy once the pair gave up
              fence_proxy_async();
              issue_half<BITS, GRP>(p, ps, stage, pr.seg.b, pr.seg.h, pr.j, slen, true, extra_tx(true));
              ++*issued;
              ++pr.j;
              *cur = prod_settle<kSlot>(pr, pre, slen, p.B, H, cr);
            }
          }
        } else if (k > 0 && prod.valid) {
          // refill the stage of the previous block once the V-warp has
          // released it: its reads of the stage happen before its arrive on
          // `other`, which this wait acquires, so the copy cannot overtake them
          const uint32_t kp = k - 1;
          const int sp = static_cast<int>(kp % kS);
          // no new copy once the pair gave up: it drains what it issued
          if (wait_bar(&ps.other[sp], (kp / kS) & 1u, p.err, abort, p.wait_ns)) {
            if (lane == 0) {
              issue_block<BITS, GRP>(p, ps, sp, prod.seg.b, prod.seg.h, prod.j, slen, extra_tx(true));
              ++*issued;
            }
            ++prod.j;
            prod = prod_settle<kSlot>(prod, pre, slen, p.B, H, cr);
          }
        }
      }
    } else {
      // ===================== V-warp: softmax and values =====================
      u64 u[kG][8];
      float m[kG], z[kG];                               // z: per token-lane
#pragma unroll
      for (int hh = 0; hh < kG; ++hh) {
        m[hh] = -INFINITY;
        z[hh] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) u[hh][i] = 0ull;
      }
      const int g = cs >> 1;                            // V group of channels 16cs..16cs+15
      for (int j = seg.jb; j < seg.je; ++j, ++k) {
        const int stage = static_cast<int>(k % kS);
        const int pb = static_cast<int>(k & 1u);
        if (*abort) {                                    // a wait of this pair ran out
          alive = false;
          break;
        }
        wait_bar(kSplit ? &ps.other[stage] : &ps.full[stage], (k / kS) & 1u, p.err, abort, p.wait_ns);
        wait_bar(&ps.pfull[pb], (k >> 1) & 1u, p.err, abort, p.wait_ns);
        const Stage& st = ps.st[stage];
        const int nvalid = min(kTB, len - j * kTB);

        // scores of token `lane`: sum the eight channel-slice partials
        u64 s01 = 0ull, s23 = 0ull;                     // heads (0, 1) and (2, 3)
        const float* part = ps.part[pb];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const ulonglong2 v = *reinterpret_cast<const ulonglong2*>(part + part_index(lane, i));
          s01 = add2(s01, v.x);
          s23 = add2(s23, v.y);
        }
        float s[kG] = {lo_f(s01), hi_f(s01), lo_f(s23), hi_f(s23)};
        __syncwarp();
        if (lane == 0) mbar_arrive(&ps.pempty[pb]);

        // online softmax over the block (log2 units).  The reference m of a
        // head moves only when a block's maximum exceeds it by more than
        // kLazy (always on the first block, where m = -inf); otherwise the
        // block's exponentials are taken against the old reference and stay
        // below 2^kLazy.  Any reference gives the same u / z in exact
        // arithmetic (the block rule with a stale but consistent m), and the
        // partials carry the reference the merge rescales by.
        const bool valid = lane < nvalid;
        float pr[kG], bm[kG];
        bool grow = false;
#pragma unroll
        for (int hh = 0; hh < kG; ++hh) {
          s[hh] = valid ? s[hh] : -INFINITY;
          bm[hh] = warp_max(s[hh]);
          grow |= bm[hh] > m[hh] + kLazy;
        }
        if (grow) {                                     // warp-uniform
#pragma unroll
          for (int hh = 0; hh < kG; ++hh) {
            const float mn = fmaxf(m[hh], bm[hh]);
            const float a = ex2(m[hh] - mn);            // 0 on the first block (m = -inf)
            z[hh] *= a;
            m[hh] = mn;
            const u64 a2 = pack2(a, a);
#pragma unroll
            for (int i = 0; i < 8; ++i) u[hh][i] = mul2(u[hh][i], a2);
          }
        }
#pragma unroll
        for (int hh = 0; hh < kG; ++hh) {
          pr[hh] = valid ? ex2(s[hh] - m[hh]) : 0.f;
          z[hh] += pr[hh];
        }
        if (GRP == 32) {
          // p' = p * s_v of this lane's token for each V group, as (p', p') pairs
          const float4 sv = *reinterpret_cast<const float4*>(st.vs[lane]);
          const float svg[4] = {sv.x, sv.y, sv.z, sv.w};
          const u64 p01 = pack2(pr[0], pr[1]), p23 = pack2(pr[2], pr[3]);
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            const float sg = valid ? svg[gg] : 0.f;
            const u64 s2 = pack2(sg, sg);
            *reinterpret_cast<ulonglong2*>(&ps.pv[lane][4 * gg]) =
                make_ulonglong2(mul2(p01, s2), mul2(p23, s2));
          }
        } else {
          // g8: p itself; the V scales go on the codes
          *reinterpret_cast<float4*>(&ps.pv[lane][0]) = make_float4(pr[0], pr[1], pr[2], pr[3]);
        }
        __syncwarp();

        // values: lane (ts, cs), token 4*it + ts, channels 16cs..16cs+15
#pragma unroll 2
        for (int it = 0; it < kTB / 4; ++it) {
          const int t = block_token<GRP>(it, ts);
          const float4 p4 = *reinterpret_cast<const float4*>(&ps.pv[t][GRP == 32 ? 4 * g : 0]);
          // (code - qmax) eps exactly, so a zero code contributes exactly zero
          u64 f[8];
          v_offsets<BITS>(st.vc, t, cs, f);
          const u64 pp[kG] = {pack2(p4.x, p4.x), pack2(p4.y, p4.y), pack2(p4.z, p4.z),
                              pack2(p4.w, p4.w)};
          if (GRP == 8) {
            // the scales of V groups 2 cs and 2 cs + 1 (channels 16 cs .. +7,
            // +8 .. +15); zero past the length, where the stage holds stale
            // scales and p is already zero
            const float2 sv = *reinterpret_cast<const float2*>(&st.vs[t][2 * cs]);
            const bool tv = t < nvalid;
            const u64 s0 = pack2(tv ? sv.x : 0.f, tv ? sv.x : 0.f), s1 = pack2(tv ? sv.y : 0.f, tv ? sv.y : 0.f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              f[i] = mul2(f[i], s0);
              f[4 + i] = mul2(f[4 + i], s1);
            }
          }
#pragma unroll
          for (int hh = 0; hh < kG; ++hh)
#pragma unroll
            for (int i = 0; i < 8; ++i) u[hh][i] = fma2(pp[hh], f[i], u[hh][i]);
        }
        __syncwarp();
        if constexpr (kSplit) {
          // this warp has read the stage's V half for the last time: refill it
          if (lane == 0) {
            Prod pr = *cur;
            if (pr.valid && !*abort) {                   // no new copy once the pair gave up
              fence_proxy_async();
              issue_half<BITS, GRP>(p, ps, stage, pr.seg.b, pr.seg.h, pr.j, slen, false, 0u);
              ++*issued;
              ++pr.j;
              *cur = prod_settle<kSlot>(pr, pre, slen, p.B, H, cr);
            }
          }
        } else if (lane == 0) {
          mbar_arrive(&ps.other[stage]);               // the S-warp may refill the stage
        }
      }

      if (!alive) break;
      if (kSlot && seg.jb >= seg.je) {                 // the append slot alone: no state
        first = false;
        seg = next_seg<kSlot>(seg, pre, slen, p.B, H, cr);
        continue;
      }
      // the pair's state for the segment: z summed over the token lanes, u
      // over the four token groups; lanes with ts = 0 hold channels 16cs..
#pragma unroll
      for (int hh = 0; hh < kG; ++hh) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z[hh] += __shfl_xor_sync(0xffffffffu, z[hh], o);
      }
      const bool whole = (seg.jb == 0) && (seg.je == seg_blocks<kSlot>(seg, slen)) && !p.force_partial;
      const long long slot = static_cast<long long>(worker) + head;
#pragma unroll
      for (int hh = 0; hh < kG; ++hh) {
        float uf[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          // u carries the factor eps of its slot: scale it back
          float x = lo_f(u[hh][i]) * VSlot<BITS>::inv_eps(2 * i);
          float y = hi_f(u[hh][i]) * VSlot<BITS>::inv_eps(2 * i + 1);
          x += __shfl_xor_sync(0xffffffffu, x, 8);
          y += __shfl_xor_sync(0xffffffffu, y, 8);
          x += __shfl_xor_sync(0xffffffffu, x, 16);
          y += __shfl_xor_sync(0xffffffffu, y, 16);
          uf[2 * i] = x;
          uf[2 * i + 1] = y;
        }
        if (ts != 0) continue;
        if (whole) {
          // the worker covered the whole (b, h): O = u / z
          const float iz = 1.f / z[hh];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            store_from_f32(p.O, (qrow + hh) * kD + 16 * cs + c, uf[c] * iz, p.q_dtype);
        } else {
          float* part = p.partials + (slot * kG + hh) * (kD + 2);
          if (cs == 0) {
            part[0] = m[hh] * kLn2;
            part[1] = z[hh];
          }
          // 8-byte stores: the row of kD + 2 floats keeps only 8-byte alignment
          float2* dst = reinterpret_cast<float2*>(part + 2 + 16 * cs);
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[q] = make_float2(uf[2 * q], uf[2 * q + 1]);
        }
      }
    }
    first = false;
    seg = next_seg<kSlot>(seg, pre, slen, p.B, H, cr);
  }
  if (!alive && lane == 0) {
    // a wait ran out: nothing of this pair's segment is written; copies this
    // warp issued whose completion it has not seen are waited for (bounded)
    // so none still writes shared memory when the CTA exits
    // at most kS copies of a warp are in flight, the last kS it issued (a
    // phase that already completed passes at once)
    const bool issuer = kSplit || is_s;
    const uint32_t n = *issued;
    for (uint32_t kk = n > kS ? n - kS : 0; issuer && kk < n; ++kk)
      drain_bar(kSplit && !is_s ? &ps.other[kk % kS] : &ps.full[kk % kS], (kk / kS) & 1u);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Shared memory one CTA may use so that `per_sm` of them fit an SM (228 KB
// per SM, 1 KB of it reserved per CTA, at most 227 KB per CTA).
constexpr size_t smem_limit(int per_sm) { return per_sm == 1 ? 227 * 1024 : 113 * 1024; }

// The instantiation for a call's code width and group size: its launch shape
// and kernel.
struct DecodeVariant {
  int pairs, per_sm, threads;
  size_t (*smem)(int B);
  void (*kernel)(DecodeParams);
  void (*kernel_append)(DecodeParams);
};

template <int BITS, int GRP>
DecodeVariant variant_of() {
  return {Tr<BITS, GRP>::kNP, Tr<BITS, GRP>::kCtasPerSm, Tr<BITS, GRP>::kThreads, smem_bytes<BITS, GRP>,
          decode_kernel<BITS, GRP, false>, decode_kernel<BITS, GRP, true>};
}

DecodeVariant variant(const AttendArgs& a) {
  if (a.g.group == 32) return a.g.bits == 4 ? variant_of<4, 32>() : variant_of<8, 32>();
  return a.g.bits == 4 ? variant_of<4, 8>() : variant_of<8, 8>();
}

bool decode_applies(const AttendArgs& a) {
  if (!((a.g.bits == 4 || a.g.bits == 8) && (a.g.group == 32 || a.g.group == 8) && a.g.D == kD &&
        a.Lq == 1 && a.H_q == kG * a.g.H_kv))
    return false;
  const DecodeVariant v = variant(a);
  return v.smem(a.g.B) <= smem_limit(v.per_sm);
}

int decode_ctas(const AttendArgs& a) {
  const long long t_max = static_cast<long long>(a.g.B) * a.g.H_kv * ((a.g.N_cap + kTB - 1) / kTB);
  const int per_sm = variant(a).per_sm;
  long long ctas = a.splits > 0 ? a.splits : static_cast<long long>(per_sm) * (sm_count() > 0 ? sm_count() : 148);
  if (ctas > t_max) ctas = t_max;
  if (ctas < 1) ctas = 1;
  return static_cast<int>(ctas);
}

// Warp pairs per CTA: each pair is one worker of the plan.
int decode_pairs(const AttendArgs& a) { return variant(a).pairs; }

size_t decode_workspace(const AttendArgs& a) {
  return with_window_slots(a, partial_slots(decode_ctas(a) * decode_pairs(a), a.g.B, a.g.H_kv),
                           kG * (kD + 2) * sizeof(float));
}

kvq_status decode_launch(const AttendArgs& a, cudaStream_t s) {
  const int ctas = decode_ctas(a);
  const DecodeVariant v = variant(a);
  const size_t smem = v.smem(a.g.B);
  auto kernel = a.K_tail_step ? v.kernel_append : v.kernel;
  const int threads = v.threads;
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kernel), smem)) return KVQ_ERR_CUDA;
  DecodeParams p{};
  p.Q = a.Q;
  p.q_dtype = a.q_dtype;
  p.k_codes = a.k_codes;
  p.k_scales = a.k_scales;
  p.v_codes = a.v_codes;
  p.v_scales = a.v_scales;
  p.lengths = a.lengths;
  p.B = a.g.B;
  p.H = a.g.H_kv;
  p.N_cap = a.g.N_cap;
  p.k_codes_head = static_cast<long long>(a.g.k_codes_head);
  p.k_scales_head = static_cast<long long>(a.g.k_scales_head);
  p.v_codes_head = static_cast<long long>(a.g.v_codes_head);
  p.v_scales_head = static_cast<long long>(a.g.v_scales_head);
  p.qscale = a.scale * kLog2e;
  p.O = a.O;
  p.partials = static_cast<float*>(a.workspace);
  p.ctas = ctas;
  p.force_partial = a.win_lengths != nullptr;
  p.err = error_word();
  if (!p.err) return KVQ_ERR_CUDA;
  p.wait_ns = a.test_wait_ns ? a.test_wait_ns : 2000000000ull;
  p.k_tail = a.K_tail_step;
  p.v_new = a.V_new_step;
  p.in_dtype = a.step_dtype;
  p.lose_worker = a.test_lose_block >= 0 ? 0 : -1;
  p.lose_block = a.test_lose_block;
  const cudaError_t le = launch_pdl(kernel, dim3(ctas), dim3(threads), smem, s, p);
  if (le != cudaSuccess) return KVQ_ERR_CUDA;
  count_launch();

  MergeArgs m{};
  m.partials = p.partials;
  m.lengths = a.lengths;
  m.O = a.O;
  m.o_dtype = a.q_dtype;
  m.B = a.g.B;
  m.H_kv = a.g.H_kv;
  m.N_cap = a.g.N_cap;
  m.BT = kTB;
  m.ctas = ctas * decode_pairs(a);
  m.R = kG;
  m.R_pad = kG;
  m.D = kD;
  m.G = kG;
  m.Lq = 1;
  m.extra_slots = (a.K_tail_step && a.g.bits == 4) ? 1 : 0;   // the decode kernel's kSlot
  const kvq_status ws = add_window(a, p.partials, static_cast<long long>(partial_slots(m.ctas, a.g.B, a.g.H_kv)),
                                   kG * (kD + 2), kD + 2, 32 * (kD + 2), 1, &m, s);
  if (ws != KVQ_OK) return ws;
  return launch_merge(m, s);
}

const AttendImpl kDecode{"decode_gqa4_d128", decode_applies, decode_workspace, decode_launch};

}  // namespace

const AttendImpl* decode_attend_impl() { return &kDecode; }

}  // namespace kvq
