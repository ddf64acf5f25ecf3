// Multi-query chunk attention on the tcgen05 tensor cores: D = 128, 4- or 8-bit
// codes in groups of 32, bf16 Q/O, 128 or 256 query rows per KV head (the
// GQA group's heads times the chunk's queries), non-causal over the whole
// valid cache ("注意力分塊：不保存完整分數矩陣，如何保持結果？", opening section: the
// queries read the whole existing context).
//
// Per 128-token block the packed K/V bytes are decoded -- (code - qmax) *
// scale, as "KV分组打包：4-bit到底省了多少？" section "一个字节里到底装了什么"
// defines it -- into bf16 tiles in shared memory, S = Q K^T runs on the
// tensor cores into tensor memory (TMEM), the online softmax turns S into P
// in place, and O += P V runs on the tensor cores again with P read straight
// from TMEM.  The running (m, z, u) rule of "Block KV decoding: less workspace,
// more time" (section "Do not average independently normalized blocks") is
// applied per query row; u lives in TMEM.
//
// Rescaling is lazy: a row's reference maximum only moves (and O, z are
// multiplied by exp(m_old - m_new)) when a block's maximum exceeds it by more
// than 8 in log2 units.  Any reference that never falls more than that below
// the true running maximum gives the same u / z in exact arithmetic, and the
// exponentials stay <= 2^8, well inside bf16/fp32 range.
//
// Warp roles (20 warps, 96 registers each):
//   0        producer: cp.async.bulk of the packed codes + scales, one unit
//            per K or V half of a block, into a ring of 54 KB (5 units at
//            4 bits, 3 at 8 bits).  Unit order K(0), K(1), V(0), K(2), V(1),
//            ...: the K decode runs one block ahead of the V decode.
//   1        MMA issuer (one thread) and TMEM owner (512 columns)
//   2        Q loader: a 2-D TMA copy with 128-byte swizzle of the segment's
//            Q rows, once the previous segment's Q K^T products are done
//   4..7     softmax of query rows 0..127 (TMEM lanes 0..127, warp w owns
//            lanes 32*(w%4)..+31); 8..11 the same for rows 128..255
//   12..19   decode: warp w converts the 16-token slice w-12 of each K unit
//            (into one of two K tiles) and the same tokens of each V unit
//   3        idle
// The MMA order per block k is QK0(k) QK1(k) | PV0(k) QK0(k+1) PV1(k)
// QK1(k+1) | ...: while one row tile is in the softmax the tensor cores work
// on the other.  A Q K^T product overwrites the S columns that hold the
// previous block's P, so it waits for that tile's P V product to complete.
//
// TMEM columns: S/P of row tile t at [128 t, 128 t + 128), O of row tile t at
// [256 + 128 t, 256 + 128 t + 128).  P (bf16) overwrites the first 64 columns
// of its S tile.
//
// Shared memory tiles use the 128-byte-swizzled UMMA layout: a row of 64 bf16
// (128 B) with its 16-byte chunks XOR-permuted by (row % 8), eight-row atoms
// of 1 KB -- the layout a TMA copy with 128-byte swizzle writes.  Q tiles and
// the K tiles are K-major (rows = query rows / tokens, contiguous = features);
// the V tile is stored the same way (rows = tokens) and read as an MN-major
// operand.  Each 128-feature row is split in two 64-feature halves of 16 KB.
#include <cuda.h>

#include "f32x2.cuh"
#include "kvq_internal.cuh"
#include "plan.cuh"
#include "tc_common.cuh"

namespace kvq {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kBT = 128;              // tokens per block
constexpr int kThreads = 640;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLazy = 8.f;          // log2 units a row max may outrun its reference

// shared-memory carve (bytes from a 1024-aligned base)
constexpr int kTileHalf = kBT * 128;              // 16 KB: 128 rows x 64 bf16
constexpr int kOffQ = 0;                          // 2 row tiles x 2 halves
constexpr int kOffK = 4 * kTileHalf;              // 2 K tiles (double buffer)
constexpr int kOffV = kOffK + 4 * kTileHalf;      // 1 V tile
constexpr int kOffRing = kOffV + 2 * kTileHalf;   // 160 KB
constexpr int kRingBytes = 54 * 1024;
constexpr int kMaxUnits = 5;
constexpr int kOffBar = kOffRing + kRingBytes;
constexpr int kNumBars = 24;
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // TMEM base slot
constexpr int kOffPre = kOffMisc + 16;            // int pre[B + 1], len[B]

enum Bar {
  RING_FULL = 0,                 // [kMaxUnits]
  RING_EMPTY = 5,                // [kMaxUnits]
  K_READY = 10,                  // [2]
  K_FREE = 12,                   // [2]
  V_READY = 14,
  V_FREE = 15,
  Q_READY = 16,
  Q_FREE = 17,
  S_FULL = 18,                   // [2]
  P_FULL = 20,                   // [2]
  PV_DONE = 22,                  // [2]
};
constexpr int kDecodeWarps = 8;

struct ChunkParams {
  const uint8_t* k_codes;
  const float* k_scales;
  const uint8_t* v_codes;
  const float* v_scales;
  const int32_t* lengths;
  int bits, B, H, N_cap, G, Lq, R, NT;   // R = G * Lq rows per (b, h), NT = R / 128 row tiles
  long long k_codes_head, k_scales_head, v_codes_head, v_scales_head;
  float qscale;                          // scale * log2(e)
  __nv_bfloat16* O;
  float* partials;                       // [slots][R / 32][kD + 2][32]: m, z, u (feature-major)
  int ctas;
  int force_partial;                     // a window follows: no CTA writes output rows
  int causal;                            // query i of Lq reads keys [0, len - Lq + i] only
  unsigned int* err;
};

size_t smem_bytes(int B) { return 1024 + kOffPre + sizeof(int) * (2 * B + 1); }

// One K or V unit (a 128-token half-block of packed codes + scales in the
// ring) to bf16 values (code - qmax) * scale in a swizzled 128 x 128 tile.
// Warp wk converts tokens [16 wk, 16 wk + 16) -- for K half of scale group
// wk / 2, whose feature scales each lane loads once for its chunk.  Lanes
// cover consecutive 16-byte code chunks, so the code reads are conflict-free.
// The code - qmax step is exact in f32; the product with the f32 scale is
// rounded once, to bf16.  Tokens at or past nv become zeros.

// 4-bit: lane = 4 tokens x 8 chunks of 16 features (the 8-bit mapping): a
// lane's 16 features of a token are one 8-byte code load; a byte's two
// nibbles go into one f32x2 pair (nibble_pair) and one FMA makes them n - 7
// exactly.  Lanes q and q + 4 take their two 8-feature halves in opposite
// order, so a quarter warp (one token) stores to eight different bank groups.
template <bool kV>
__device__ __forceinline__ void decode_unit4(const unsigned char* u, unsigned char* dst, int wk, int lane, int nv) {
  constexpr int kCb = 64;
  const int q = lane & 7, tt = lane >> 3;
  const bool swap = (q & 4) != 0;
  const float* sc = reinterpret_cast<const float*>(u + kBT * kCb);
  u64 ks[8];                                    // slot 4 i + r: pair r of 8-feature half i ^ swap
  if (!kV) {
    if (16 * wk < nv) {
      const float4* s4 = reinterpret_cast<const float4*>(sc + (wk >> 1) * kD + 16 * q);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int ci = i ^ (swap ? 1 : 0);
        const float4 v0 = s4[2 * ci], v1 = s4[2 * ci + 1];
        ks[4 * i] = pack2(v0.x, v0.y);
        ks[4 * i + 1] = pack2(v0.z, v0.w);
        ks[4 * i + 2] = pack2(v1.x, v1.y);
        ks[4 * i + 3] = pack2(v1.z, v1.w);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) ks[i] = 0ull;
    }
  }
  const u64 mul = pack2(256.f, 16.f), add = pack2(-263.f, -23.f);
#pragma unroll 1
  for (int it = 0; it < 4; ++it) {
    const int t = 16 * wk + 4 * it + tt;
    uint4 o[2];
    if (t < nv) {
      const uint2 w2 = *reinterpret_cast<const uint2*>(u + t * kCb + 8 * q);
      const uint32_t w[2] = {swap ? w2.y : w2.x, swap ? w2.x : w2.y};
      u64 s2 = 0ull;
      if (kV) {
        const float s = sc[4 * t + (q >> 1)];
        s2 = pack2(s, s);
      }
      uint32_t h[8];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const u64 f = fma2(nibble_pair(byte_at15(w[i], r)), mul, add);
          const u64 x = mul2(f, kV ? s2 : ks[4 * i + r]);
          h[4 * i + r] = pack_bf16(lo_f(x), hi_f(x));
        }
      }
      o[0] = make_uint4(h[0], h[1], h[2], h[3]);
      o[1] = make_uint4(h[4], h[5], h[6], h[7]);
    } else {
      o[0] = make_uint4(0u, 0u, 0u, 0u);
      o[1] = o[0];
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int ch = 2 * q + (i ^ (swap ? 1 : 0));
      *reinterpret_cast<uint4*>(dst + (ch >> 3) * kTileHalf + swz(t, ch & 7)) = o[i];
    }
  }
}

// 8-bit: lane = 4 tokens x 8 chunks of 16 features; two bytes go into the
// low mantissa bits of an f32x2 pair of 2^23, one add makes them c - 127.
// Lanes q and q + 4 store their two 16-byte chunks in opposite order, so a
// quarter warp (one token) stores to eight different bank groups.
template <bool kV>
__device__ __forceinline__ void decode_unit8(const unsigned char* u, unsigned char* dst, int wk, int lane, int nv) {
  constexpr int kCb = 128;
  const int q = lane & 7, tt = lane >> 3;
  const bool swap = (q & 4) != 0;
  const float* sc = reinterpret_cast<const float*>(u + kBT * kCb);
  u64 ks[8];                                    // slot 4 i + r: pair r of chunk i ^ swap
  if (!kV) {
    if (16 * wk < nv) {
      const float4* s4 = reinterpret_cast<const float4*>(sc + (wk >> 1) * kD + 16 * q);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int ci = i ^ (swap ? 1 : 0);
        const float4 v0 = s4[2 * ci], v1 = s4[2 * ci + 1];
        ks[4 * i] = pack2(v0.x, v0.y);
        ks[4 * i + 1] = pack2(v0.z, v0.w);
        ks[4 * i + 2] = pack2(v1.x, v1.y);
        ks[4 * i + 3] = pack2(v1.z, v1.w);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) ks[i] = 0ull;
    }
  }
  const u64 sub = pack2(-8388735.f, -8388735.f);
#pragma unroll 1
  for (int it = 0; it < 4; ++it) {
    const int t = 16 * wk + 4 * it + tt;
    uint4 o[2];
    if (t < nv) {
      const uint4 w4 = *reinterpret_cast<const uint4*>(u + t * kCb + 16 * q);
      const uint32_t w[4] = {swap ? w4.z : w4.x, swap ? w4.w : w4.y, swap ? w4.x : w4.z, swap ? w4.y : w4.w};
      u64 s2 = 0ull;
      if (kV) {
        const float s = sc[4 * t + (q >> 1)];
        s2 = pack2(s, s);
      }
      uint32_t h[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int r = 0; r < 4; r += 2) {
          const u64 f = add2(byte_pair(w[i], r), sub);
          const u64 x = mul2(f, kV ? s2 : ks[2 * i + r / 2]);
          h[2 * i + r / 2] = pack_bf16(lo_f(x), hi_f(x));
        }
      }
      o[0] = make_uint4(h[0], h[1], h[2], h[3]);
      o[1] = make_uint4(h[4], h[5], h[6], h[7]);
    } else {
      o[0] = make_uint4(0u, 0u, 0u, 0u);
      o[1] = o[0];
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int ch = 2 * q + (i ^ (swap ? 1 : 0));
      *reinterpret_cast<uint4*>(dst + (ch >> 3) * kTileHalf + swz(t, ch & 7)) = o[i];
    }
  }
}

// Maximum (kMin: minimum) of 64 raw scores held in registers, as eight
// independent three-input chains.
template <bool kMin>
__device__ __forceinline__ float row_extreme(const uint32_t (&sr)[64]) {
  auto f = [](uint32_t x) { return __uint_as_float(x); };
  auto op3 = [](float a, float b, float c) { return kMin ? min3(a, b, c) : max3(a, b, c); };
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    acc[j] = op3(f(sr[j]), f(sr[8 + j]), f(sr[16 + j]));        // columns 0..23
    acc[j] = op3(acc[j], f(sr[24 + j]), f(sr[32 + j]));         // 24..39
    acc[j] = op3(acc[j], f(sr[40 + j]), f(sr[48 + j]));         // 40..55
  }
  const float a = op3(acc[0], acc[1], acc[2]);
  const float b = op3(acc[3], acc[4], acc[5]);
  const float c = op3(acc[6], acc[7], a);
  float r = op3(b, c, f(sr[56]));
#pragma unroll
  for (int j = 57; j < 64; j += 2) r = op3(r, f(sr[j]), f(sr[j + 1 < 64 ? j + 1 : j]));   // 56..63
  return r;
}

// One instantiation per code width, so each carries one decode path only
// (a smaller body for the instruction cache the 20 warp roles share).
template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) chunk_kernel(const __grid_constant__ CUtensorMap qmap, ChunkParams p) {
  griddep_wait();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = su(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  unsigned char* sm = smem_raw + (base - raw_addr);
  int* pre = reinterpret_cast<int*>(sm + kOffPre);
  int* slen = pre + p.B + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);
  const uint32_t bar0 = base + kOffBar;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.H;
  constexpr int cb = kD * BITS / 8;                       // code bytes per token
  const int unit_bytes = kBT * cb + 2048;                 // codes + scales of a K or V half-block
  const uint32_t nu = static_cast<uint32_t>(min(kMaxUnits, kRingBytes / unit_bytes));

  if (warp == 0) warp_block_prefix(p.lengths, p.B, p.N_cap, kBT, pre);
  for (int b = threadIdx.x; b < p.B; b += kThreads) slen[b] = clamp_len(p.lengths[b], p.N_cap);
  if (threadIdx.x == 32) {
    *abort_flag = 0;
    for (uint32_t u = 0; u < nu; ++u) {
      mbar_init(bar(RING_FULL + u), 1);
      mbar_init(bar(RING_EMPTY + u), kDecodeWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(K_READY + i), kDecodeWarps);
      mbar_init(bar(K_FREE + i), 1);
      mbar_init(bar(S_FULL + i), 1);
      mbar_init(bar(P_FULL + i), 4);
      mbar_init(bar(PV_DONE + i), 1);
    }
    mbar_init(bar(V_READY), kDecodeWarps);
    mbar_init(bar(V_FREE), 1);
    mbar_init(bar(Q_READY), 1);
    mbar_init(bar(Q_FREE), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + kOffMisc),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + kOffMisc);

  // sequences with a length outside 1..N_cap: report; rows of sequences with
  // no valid key are zero (no block of theirs exists).  With a window the
  // merge owns both.
  for (int b = p.force_partial ? p.B : blockIdx.x; b < p.B; b += gridDim.x) {
    const int raw = p.lengths[b];
    if (threadIdx.x == 0 && (raw < 1 || raw > p.N_cap)) record_error(p.err, KVQ_ERR_LENGTH);
    if (slen[b] == 0) {
      const long long row0 = static_cast<long long>(b) * H * p.R;
      for (long long i = threadIdx.x; i < static_cast<long long>(H) * p.R * kD; i += kThreads)
        p.O[row0 * kD + i] = __float2bfloat16_rn(0.f);
    }
  }

  const CtaRange cr = cta_range(pre, p.B, H, p.ctas, blockIdx.x);
  if (cr.g0 < cr.g1) {
    if (warp == 0) {
      // ======================= producer =======================
      if (lane == 0) {
        Cursor kc, vc;
        kc.start(pre, p.B, H, cr);
        vc.start(pre, p.B, H, cr);
        uint32_t n = 0;
        auto unit = [&](const Cursor& c, bool is_v) {
          const uint32_t slot = n % nu;
          if (n >= nu) wait_bar(bar(RING_EMPTY + slot), ((n / nu) - 1) & 1u, p.err, abort_flag);
          const long long head = static_cast<long long>(c.seg.b) * H + c.seg.h;
          const int t0 = c.j * kBT;
          const int nv = min(kBT, slen[c.seg.b] - t0);
          const uint32_t dst = base + kOffRing + slot * unit_bytes;
          const uint32_t fb = bar(RING_FULL + slot);
          if (!is_v) {
            const int ng = (nv + 31) / 32;
            mbar_expect_tx(fb, static_cast<uint32_t>(nv * cb + ng * kD * 4));
            bulk_g2s(dst, p.k_codes + head * p.k_codes_head + static_cast<long long>(t0) * cb, nv * cb, fb);
            bulk_g2s(dst + kBT * cb, p.k_scales + head * p.k_scales_head + static_cast<long long>(t0 / 32) * kD,
                     ng * kD * 4, fb);
          } else {
            mbar_expect_tx(fb, static_cast<uint32_t>(nv * cb + nv * 16));
            bulk_g2s(dst, p.v_codes + head * p.v_codes_head + static_cast<long long>(t0) * cb, nv * cb, fb);
            bulk_g2s(dst + kBT * cb, p.v_scales + head * p.v_scales_head + static_cast<long long>(t0) * 4, nv * 16,
                     fb);
          }
          ++n;
        };
        if (kc.valid) {
          unit(kc, false);
          kc.next(pre, p.B, H, cr);
        }
        while (vc.valid) {
          if (kc.valid) {
            unit(kc, false);
            kc.next(pre, p.B, H, cr);
          }
          unit(vc, true);
          vc.next(pre, p.B, H, cr);
        }
      }
    } else if (warp == 1) {
      // ======================= MMA issuer =======================
      if (lane == 0) {
        const uint32_t idesc_qk = instr_desc(kBT, false);
        const uint32_t idesc_pv = instr_desc(kD, true);
        auto qk = [&](int t, uint32_t k) {
          const uint32_t kt = base + kOffK + (k & 1u) * 2 * kTileHalf;
          for (int i = 0; i < kD / 16; ++i) {
            const uint32_t q_addr = base + kOffQ + t * 2 * kTileHalf + (i >> 2) * kTileHalf + (i & 3) * 32;
            const uint32_t k_addr = kt + (i >> 2) * kTileHalf + (i & 3) * 32;
            mma_ss(tmem + 128u * t, smem_desc(q_addr, 16, 1024), smem_desc(k_addr, 16, 1024), idesc_qk, i > 0);
          }
          mma_commit(bar(S_FULL + t));
        };
        auto pv = [&](int t, uint32_t k, bool first) {
          wait_bar(bar(P_FULL + t), k & 1u, p.err, abort_flag);
          tc_fence_after();
          for (int i = 0; i < kBT / 16; ++i) {
            const uint32_t v_addr = base + kOffV + i * 16 * 128;
            mma_ts(tmem + 256u + 128u * t, tmem + 128u * t + 8u * i, smem_desc(v_addr, kTileHalf, 1024), idesc_pv,
                   (!first) || (i > 0));
          }
          mma_commit(bar(PV_DONE + t));
        };
        Cursor c;
        c.start(pre, p.B, H, cr);
        uint32_t sq = 0;
        // block 0: Q of the first segment, its K tile, both Q K^T products
        wait_bar(bar(Q_READY), sq & 1u, p.err, abort_flag);
        ++sq;
        wait_bar(bar(K_READY), 0u, p.err, abort_flag);
        tc_fence_after();
        for (int t = 0; t < p.NT; ++t) qk(t, 0);
        mma_commit(bar(K_FREE));
        if (c.last()) mma_commit(bar(Q_FREE));
        Cursor cn = c;
        cn.next(pre, p.B, H, cr);
        for (uint32_t k = 0; c.valid; ++k) {
          const bool boundary = cn.valid && cn.first();
          wait_bar(bar(V_READY), k & 1u, p.err, abort_flag);
          tc_fence_after();
          pv(0, k, c.first());
          if (cn.valid && !boundary) {
            wait_bar(bar(K_READY + ((k + 1) & 1u)), ((k + 1) >> 1) & 1u, p.err, abort_flag);
            wait_bar(bar(PV_DONE), k & 1u, p.err, abort_flag);
            tc_fence_after();
            qk(0, k + 1);
          }
          if (p.NT == 2) pv(1, k, c.first());
          mma_commit(bar(V_FREE));
          if (cn.valid) {
            if (boundary) {
              wait_bar(bar(Q_READY), sq & 1u, p.err, abort_flag);
              ++sq;
              wait_bar(bar(K_READY + ((k + 1) & 1u)), ((k + 1) >> 1) & 1u, p.err, abort_flag);
              wait_bar(bar(PV_DONE), k & 1u, p.err, abort_flag);
              tc_fence_after();
              qk(0, k + 1);
            }
            if (p.NT == 2) {
              wait_bar(bar(PV_DONE + 1), k & 1u, p.err, abort_flag);
              tc_fence_after();
              qk(1, k + 1);
            }
            mma_commit(bar(K_FREE + ((k + 1) & 1u)));
            if (cn.last()) mma_commit(bar(Q_FREE));
          }
          c = cn;
          cn.next(pre, p.B, H, cr);
        }
      }
      __syncwarp();
    } else if (warp == 2) {
      // ======================= Q loader =======================
      if (lane == 0) {
        uint32_t s = 0;
        for (Seg seg = first_seg(pre, p.B, H, cr); seg.valid; seg = next_seg(seg, pre, p.B, H, cr), ++s) {
          if (s > 0) wait_bar(bar(Q_FREE), (s - 1) & 1u, p.err, abort_flag);
          const int row0 = (seg.b * H * p.G + seg.h * p.G) * p.Lq;
          mbar_expect_tx(bar(Q_READY), static_cast<uint32_t>(p.NT * 2 * kTileHalf));
          for (int t = 0; t < p.NT; ++t)
            for (int half = 0; half < 2; ++half)
              tma_load_2d(base + kOffQ + (2 * t + half) * kTileHalf, &qmap, 64 * half, row0 + 128 * t, bar(Q_READY));
        }
      }
    } else if (warp >= 12) {
      // ======================= decode K/V to bf16 tiles =======================
      const int wk = warp - 12;                          // 16-token slice of each unit
      Cursor kc, vc;
      kc.start(pre, p.B, H, cr);
      vc.start(pre, p.B, H, cr);
      uint32_t n = 0, kb = 0, vb = 0;
      auto decode = [&](const Cursor& c, bool is_v) {
        const uint32_t slot = n % nu;
        wait_bar(bar(RING_FULL + slot), (n / nu) & 1u, p.err, abort_flag);
        if (!is_v && kb >= 2) wait_bar(bar(K_FREE + (kb & 1u)), ((kb >> 1) - 1) & 1u, p.err, abort_flag);
        if (is_v && vb >= 1) wait_bar(bar(V_FREE), (vb - 1) & 1u, p.err, abort_flag);
        const unsigned char* u = sm + kOffRing + slot * unit_bytes;
        unsigned char* dst = sm + (is_v ? kOffV : kOffK + (kb & 1u) * 2 * kTileHalf);
        const int nv = min(kBT, slen[c.seg.b] - c.j * kBT);
        if constexpr (BITS == 4) {
          if (is_v) decode_unit4<true>(u, dst, wk, lane, nv);
          else decode_unit4<false>(u, dst, wk, lane, nv);
        } else {
          if (is_v) decode_unit8<true>(u, dst, wk, lane, nv);
          else decode_unit8<false>(u, dst, wk, lane, nv);
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(is_v ? V_READY : K_READY + (kb & 1u)));
          mbar_arrive(bar(RING_EMPTY + slot));
        }
        ++n;
        if (is_v) ++vb; else ++kb;
      };
      if (kc.valid) {
        decode(kc, false);
        kc.next(pre, p.B, H, cr);
      }
      while (vc.valid) {
        if (kc.valid) {
          decode(kc, false);
          kc.next(pre, p.B, H, cr);
        }
        decode(vc, true);
        vc.next(pre, p.B, H, cr);
      }
    } else if (warp >= 4) {
      // ======================= softmax: one query row per thread =======================
      const int tile = (warp - 4) >> 2;
      const int r = ((warp & 3) << 5) + lane;            // TMEM lane = row within the tile
      const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const uint32_t s_col = tmem + lane_addr + 128u * tile;
      const uint32_t o_col = tmem + lane_addr + 256u + 128u * tile;
      const bool neg = p.qscale < 0.f;
      const float aq = fabsf(p.qscale);
      // the row's query index within its head (rows are head-major, Lq each)
      const int qi = (128 * tile + r) % p.Lq;
      if (tile < p.NT) {
        float m_ref = -INFINITY, z = 0.f;
        Cursor c;
        c.start(pre, p.B, H, cr);
        for (uint32_t k = 0; c.valid; ++k, c.next(pre, p.B, H, cr)) {
          if (c.first()) {
            m_ref = -INFINITY;
            z = 0.f;
          }
          wait_bar(bar(S_FULL + tile), k & 1u, p.err, abort_flag);
          tc_fence_after();
          // valid columns of this row: the sequence end, and with a causal
          // mask the row's own position (none at all if this block starts
          // after it; m_ref then stays -inf and every p is zero)
          const int nv_seq = min(kBT, slen[c.seg.b] - c.j * kBT);
          const int nv = p.causal ? min(nv_seq, slen[c.seg.b] - p.Lq + qi + 1 - c.j * kBT) : nv_seq;
          // pass 1: the row's extreme over the valid columns, 64 at a time
          float mx = neg ? INFINITY : -INFINITY;
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t sr[64];
            KVQ_LD32_AT(sr, 0, s_col + 64u * hh);
            KVQ_LD32_AT(sr, 32, s_col + 64u * hh + 32u);
            tmem_wait_ld();
            if (nv < kBT) {
              // tokens past the sequence end stay out of the max
              const uint32_t fill = __float_as_uint(neg ? INFINITY : -INFINITY);
#pragma unroll
              for (int e = 0; e < 64; ++e)
                if (64 * hh + e >= nv) sr[e] = fill;
            }
            mx = neg ? fminf(mx, row_extreme<true>(sr)) : fmaxf(mx, row_extreme<false>(sr));
          }
          const float mb = mx * p.qscale;
          // lazy rescale: move the reference only when the block max outruns it
          const bool need = mb > m_ref + kLazy;
          const float m_new = need ? mb : m_ref;
          const float a = need ? ex2(m_ref - m_new) : 1.f;  // 0 on the first block
          z *= a;
          m_ref = m_new;
          if (__any_sync(0xffffffffu, need) && !c.first()) {
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t orr[32];
              KVQ_LD32(orr, o_col + 32u * cc);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * a);
              KVQ_ST32(o_col + 32u * cc, orr);
            }
          }
          // pass 2: p = exp2(s * qscale - m_ref) as bf16, written over the S columns.
          // A block with every row's columns valid (all blocks but a sequence's
          // last, without the causal mask) takes a loop with no masking; the
          // choice is warp-wide because the TMEM accesses are.
          const u64 qs2 = pack2(p.qscale, p.qscale), nm2 = pack2(-m_ref, -m_ref);
          u64 z2 = 0ull;
          if (__all_sync(0xffffffffu, nv >= kBT)) {
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t sr[32];
              KVQ_LD32(sr, s_col + 32u * cc);
              tmem_wait_ld();
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const u64 x = fma2(pack2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), qs2, nm2);
                const float p0 = ex2(lo_f(x)), p1 = ex2(hi_f(x));
                z2 = add2(z2, pack2(p0, p1));
                pk[e] = pack_bf16(p0, p1);
              }
              KVQ_ST16(s_col + 16u * cc, pk);
            }
          } else {
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t sr[32];
              KVQ_LD32(sr, s_col + 32u * cc);
              tmem_wait_ld();
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const u64 x = fma2(pack2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), qs2, nm2);
                const float p0 = 32 * cc + 2 * e < nv ? ex2(lo_f(x)) : 0.f;
                const float p1 = 32 * cc + 2 * e + 1 < nv ? ex2(hi_f(x)) : 0.f;
                z2 = add2(z2, pack2(p0, p1));
                pk[e] = pack_bf16(p0, p1);
              }
              KVQ_ST16(s_col + 16u * cc, pk);
            }
          }
          z += lo_f(z2) + hi_f(z2);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(P_FULL + tile));
          if (c.last()) {
            // the segment's last P V product must be done before O is read
            wait_bar(bar(PV_DONE + tile), k & 1u, p.err, abort_flag);
            tc_fence_after();
            const bool whole = (c.seg.jb == 0) && (c.seg.je == c.seg.nb) && !p.force_partial;
            const long long head = static_cast<long long>(c.seg.b) * H + c.seg.h;
            const long long row = (static_cast<long long>(c.seg.b) * H * p.G + static_cast<long long>(c.seg.h) * p.G) *
                                      p.Lq + tile * 128 + r;
            // the slot's rows in 32-row chunks, each chunk's fields contiguous
            // (field f of row rr at (rr / 32) * (kD + 2) * 32 + f * 32 + rr % 32):
            // this warp's 32 rows are one chunk, written as 130 whole lines
            const int rr = tile * 128 + r;
            float* part = p.partials + (static_cast<long long>(blockIdx.x) + head) * (kD + 2) * p.R +
                          static_cast<long long>(rr >> 5) * (kD + 2) * 32 + (rr & 31);
            if (!whole) {
              part[0] = m_ref * kLn2;
              part[32] = z;
            }
            // z = 0: a causal row with no visible key (length < Lq, reported by the merge)
            const float inv = z > 0.f ? 1.f / z : 0.f;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t orr[32];
              KVQ_LD32(orr, o_col + 32u * cc);
              tmem_wait_ld();
              if (whole) {
                uint32_t ob[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                  ob[e] = pack_bf16(__uint_as_float(orr[2 * e]) * inv, __uint_as_float(orr[2 * e + 1]) * inv);
                uint4* dst = reinterpret_cast<uint4*>(p.O + row * kD + 32 * cc);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                  dst[qq] = make_uint4(ob[4 * qq], ob[4 * qq + 1], ob[4 * qq + 2], ob[4 * qq + 3]);
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) part[(2 + 32 * cc + e) * 32] = __uint_as_float(orr[e]);
              }
            }
            tc_fence_before();
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int rows_per_head(const AttendArgs& a) { return (a.H_q / a.g.H_kv) * a.Lq; }

bool chunk_applies(const AttendArgs& a) {
  const int R = rows_per_head(a);
  return a.g.D == kD && a.g.group == 32 && (a.g.bits == 4 || a.g.bits == 8) && a.q_dtype == KVQ_BF16 &&
         (R == 128 || R == 256) &&
         static_cast<long long>(a.g.B) * a.H_q * a.Lq < (1LL << 31) && smem_bytes(a.g.B) <= 227 * 1024;
}

int chunk_ctas(const AttendArgs& a) {
  const long long t_max = static_cast<long long>(a.g.B) * a.g.H_kv * ((a.g.N_cap + kBT - 1) / kBT);
  long long ctas = a.splits > 0 ? a.splits : (sm_count() > 0 ? sm_count() : 148);
  if (ctas > t_max) ctas = t_max;
  if (ctas < 1) ctas = 1;
  return static_cast<int>(ctas);
}

size_t chunk_workspace(const AttendArgs& a) {
  return with_window_slots(a, partial_slots(chunk_ctas(a), a.g.B, a.g.H_kv),
                           static_cast<size_t>(rows_per_head(a)) * (kD + 2) * sizeof(float));
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link)
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_tiled() {
  static EncodeTiled fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiled>(nullptr);
    return reinterpret_cast<EncodeTiled>(f);
  }();
  return fn;
}

// Q as a 2-D bf16 tensor [B * H_q * Lq rows][128], boxes of 128 rows x 64
// features written with the 128-byte swizzle the UMMA descriptors expect.
bool make_q_map(const AttendArgs& a, CUtensorMap* map) {
  const EncodeTiled enc = encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD),
                              static_cast<cuuint64_t>(a.g.B) * a.H_q * a.Lq};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.Q), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

kvq_status chunk_launch(const AttendArgs& a, cudaStream_t s) {
  const int ctas = chunk_ctas(a);
  const size_t smem = smem_bytes(a.g.B);
  auto kernel = a.g.bits == 4 ? chunk_kernel<4> : chunk_kernel<8>;
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kernel), smem)) return KVQ_ERR_CUDA;
  CUtensorMap qmap;
  if (!make_q_map(a, &qmap)) return KVQ_ERR_CUDA;
  ChunkParams p{};
  p.k_codes = a.k_codes;
  p.k_scales = a.k_scales;
  p.v_codes = a.v_codes;
  p.v_scales = a.v_scales;
  p.lengths = a.lengths;
  p.bits = a.g.bits;
  p.B = a.g.B;
  p.H = a.g.H_kv;
  p.N_cap = a.g.N_cap;
  p.G = a.H_q / a.g.H_kv;
  p.Lq = a.Lq;
  p.R = rows_per_head(a);
  p.NT = p.R / 128;
  p.k_codes_head = static_cast<long long>(a.g.k_codes_head);
  p.k_scales_head = static_cast<long long>(a.g.k_scales_head);
  p.v_codes_head = static_cast<long long>(a.g.v_codes_head);
  p.v_scales_head = static_cast<long long>(a.g.v_scales_head);
  p.qscale = a.scale * kLog2e;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.partials = static_cast<float*>(a.workspace);
  p.ctas = ctas;
  p.force_partial = a.win_lengths != nullptr;
  p.causal = a.causal;
  p.err = error_word();
  if (!p.err) return KVQ_ERR_CUDA;
  if (launch_pdl(kernel, dim3(ctas), dim3(kThreads), smem, s, qmap, p) != cudaSuccess) return KVQ_ERR_CUDA;
  count_launch();

  MergeArgs m{};
  m.partials = p.partials;
  m.lengths = a.lengths;
  m.O = a.O;
  m.o_dtype = a.q_dtype;
  m.B = a.g.B;
  m.H_kv = a.g.H_kv;
  m.N_cap = a.g.N_cap;
  m.BT = kBT;
  m.ctas = ctas;
  m.R = p.R;
  m.R_pad = p.R;
  m.D = kD;
  m.G = p.G;
  m.Lq = a.Lq;
  m.causal = a.causal;
  m.feature_major = true;
  const kvq_status ws = add_window(a, p.partials, static_cast<long long>(partial_slots(ctas, a.g.B, a.g.H_kv)),
                                   static_cast<long long>(kD + 2) * p.R, 1, static_cast<long long>(kD + 2) * 32, 32,
                                   &m, s);
  if (ws != KVQ_OK) return ws;
  return launch_merge(m, s);
}

const AttendImpl kChunk{"chunk_tcgen05_d128", chunk_applies, chunk_workspace, chunk_launch};

}  // namespace

const AttendImpl* chunk_attend_impl() { return &kChunk; }

}  // namespace kvq
