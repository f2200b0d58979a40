// Tensor-core attention kernel of ReHyAt's chunked hybrid attention for
// B200 (sm_100a): tcgen05.mma with TMEM accumulators, TMA-staged K/V tiles.
//
// Computes, for 128 query rows of one chunk (one CTA), the window softmax
// branch (a^S, n^S with stabiliser c = the row maximum), the linear branch
// a^L = phi_q(q) S^L, n^L = phi_q(q) z^L, and y = (a^S + a^L)/(n^S + n^L)
// ("ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers",
// papernotes.org note, Method, Key designs 1-4).
//
// Roles (192 threads):
//   warps 0-3  softmax / epilogue: thread r owns query row r (TMEM lane r);
//   warp 4     TMA producer (one lane): Q once, K/V tiles into 2 stages, and
//              the readout operands (phi_q weights, S^L) at the tail;
//   warp 5     MMA issuer (one lane) and TMEM owner.
// TMEM (512 columns): S double buffer [0,128) [128,256), O [256,384),
// linear numerator a^L [384,512); the phi_q pre-activation reuses [0,256)
// after the key loop.
//
// Numerics: q.k^T and P.V in bf16 with fp32 accumulation; P is rounded to
// bf16 and n^S sums the rounded values; the softmax reference point moves
// only when the running max rises by more than 2^8 (lazy rescaling) and a
// final factor exp2(m_used - m_max) makes a^S, n^S exact with respect to the
// true max c; phi_q(q) . S^L runs as tf32 with fp32 accumulation.
//
// Every wait is bounded: a barrier that does not complete within ~2 s of
// clock sets an error bit in rehyat_tc_error and the kernel unwinds.
#include <atomic>
#include <functional>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "internal.h"
#include "layout.cuh"
#include "tc_common.cuh"

namespace rehyat {

namespace {

constexpr int kD = 128;          // head width handled here
constexpr int kBM = 128;         // query rows per CTA
constexpr int kBN = 128;         // keys per tile
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;

// Shared memory map (offsets from a 1024-aligned base).  K and V have
// separate rings: a K tile is released as soon as q.k^T has read it, a V tile
// only after P.V, so the next K loads start two S-products ahead.
constexpr int kKStages = 3, kVStages = 2;
constexpr uint32_t kTileBytes = 32768;               // one 128 x 128 bf16 tile (2 boxes)
constexpr uint32_t kQOff = 0;                        // Q tile
constexpr uint32_t kKOff = 32768;                    // K ring, 3 tiles
constexpr uint32_t kVOff = kKOff + kKStages * kTileBytes;   // V ring, 2 tiles
constexpr uint32_t kPOff = kVOff + kVStages * kTileBytes;   // P tile
constexpr uint32_t kBarOff = kPOff + kTileBytes;
// Tail reuse of the K/V rings once the last P.V is done.
constexpr uint32_t kWOff = kKOff;                    // phi_q weight piece (<= 32 KB)
constexpr uint32_t kSLOff = kKOff + 32768;           // S^L piece (<= 64 KB)
constexpr uint32_t kPhiOff = kVOff;                  // phi_q(q) piece fp32 (<= 64 KB)
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;  // + alignment slack

// Barrier slots (8 bytes each).
enum {
  B_Q_FULL = 0, B_K_FULL = 1, B_K_EMPTY = 4, B_V_FULL = 7, B_V_EMPTY = 9, B_S_FULL = 11,
  B_S_FREE = 13, B_P_FULL = 15, B_PV_DONE = 16, B_TAIL_FULL = 17, B_PHI_DONE = 18,
  B_PHI_READY = 19, B_READ_DONE = 20, B_LAST_PV = 21, B_COUNT = 22
};
// A parity wait is only meaningful for a waiter at most one phase behind the
// barrier; B_LAST_PV completes exactly once (after the last P.V), so a role
// that never followed B_PV_DONE can wait on it safely.
constexpr uint32_t kTmemSlot = kBarOff + 8 * B_COUNT;       // u32: TMEM base address
constexpr uint32_t kAbortSlot = kTmemSlot + 4;              // u32: abort flag

constexpr uint32_t kColS0 = 0, kColO = 256, kColAL = 384;

}  // namespace

using namespace tc;

namespace {

// --------------------------------------------------------------- kernel
struct TcMaps {
  CUtensorMap q, k, v, rk, rv;
  CUtensorMap q8, k8;  // E4M3 copies of q, k (fp8 softmax variant)
};

struct TileSrc {
  const CUtensorMap* map_k;
  const CUtensorMap* map_v;
  int row;      // first key row within the (b, h) plane
  int nvalid;   // valid keys in this tile (<= 128)
};

__global__ void __launch_bounds__(kThreads, 1)
    tc_attn_kernel(const __grid_constant__ TcMaps maps, const AttnParams P,
                   const __nv_bfloat16* __restrict__ wq_img) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + kBarOff + 8u * i; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sbase + kAbortSlot);
  // A streaming step's fold (launched next, programmatic dependent) may start
  // once every CTA of this grid has started: it touches nothing this reads.
  asm volatile("griddepcontrol.launch_dependents;");

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int t = blockIdx.y;
  const int bh = blockIdx.z;
  const int h = bh % P.heads;

  // ---- geometry of this CTA (same rules as the CUDA-core kernel) ----
  int q_first, q_end, na, nb, a_row0;
  bool step_mode = P.seen != nullptr;
  if (!step_mode) {
    const int first = t * P.Tc;
    const int end = min(P.T, first + P.Tc);
    const int w = max(first - P.To, 0);
    q_first = first * P.HW;
    q_end = end * P.HW;
    a_row0 = w * P.HW;
    na = (end - w) * P.HW;
    nb = 0;
  } else {
    const long long seen = *P.seen;
    const int r_slices = static_cast<int>(seen < P.To ? seen : P.To);
    q_first = 0;
    q_end = P.nq_slices * P.HW;
    a_row0 = 0;
    na = r_slices * P.HW;
    nb = q_end;
  }
  const int row0 = q_first + blockIdx.x * kBM;
  if (row0 >= q_end) return;
  const int nrows = min(kBM, q_end - row0);
  const int nta = (na + kBN - 1) / kBN;
  const int ntb = (nb + kBN - 1) / kBN;
  const int nt = nta + ntb;
  const bool linear = !P.full_softmax;
  const int Dp = P.Dp;
  const int pw = piece_width(Dp);
  const int npieces = linear ? Dp / pw : 0;

  auto tile_src = [&](int j) {
    TileSrc s;
    if (j < nta) {
      s.map_k = step_mode ? &maps.rk : &maps.k;
      s.map_v = step_mode ? &maps.rv : &maps.v;
      s.row = a_row0 + j * kBN;
      s.nvalid = min(kBN, na - j * kBN);
    } else {
      const int jb = j - nta;
      s.map_k = &maps.k;
      s.map_v = &maps.v;
      s.row = jb * kBN;
      s.nvalid = min(kBN, nb - jb * kBN);
    }
    return s;
  };

  // ---- setup ----
  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      const bool by_softmax = (i == B_S_FREE || i == B_S_FREE + 1 || i == B_P_FULL ||
                               i == B_PHI_READY);
      mbar_init(bar(i), by_softmax ? kSoftmaxThreads : 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     base + kTmemSlot),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + kTmemSlot);

  if (warp == kProducerWarp) {
    // ================================================= TMA producer
    if (lane == 0) {
      bool ok = true;
      mbar_expect_tx(bar(B_Q_FULL), 2 * kBM * 128);
      tma_load_3d(base + kQOff, &maps.q, bar(B_Q_FULL), 0, row0, bh);
      tma_load_3d(base + kQOff + 16384, &maps.q, bar(B_Q_FULL), 64, row0, bh);
      for (int j = 0; j < nt && ok; ++j) {
        const TileSrc src = tile_src(j);
        const int ks = j % kKStages;
        if (j >= kKStages)
          ok = mbar_wait(bar(B_K_EMPTY + ks), ((j - kKStages) / kKStages) & 1, abort_flag, 1);
        if (!ok) break;
        const uint32_t kdst = base + kKOff + ks * kTileBytes;
        mbar_expect_tx(bar(B_K_FULL + ks), kTileBytes);
        tma_load_3d(kdst, src.map_k, bar(B_K_FULL + ks), 0, src.row, bh);
        tma_load_3d(kdst + 16384, src.map_k, bar(B_K_FULL + ks), 64, src.row, bh);
        const int vs = j & 1;
        if (j >= kVStages) ok = mbar_wait(bar(B_V_EMPTY + vs), ((j - 2) >> 1) & 1, abort_flag, 26);
        if (!ok) break;
        const uint32_t vdst = base + kVOff + vs * kTileBytes;
        mbar_expect_tx(bar(B_V_FULL + vs), kTileBytes);
        tma_load_3d(vdst, src.map_v, bar(B_V_FULL + vs), 0, src.row, bh);
        tma_load_3d(vdst + 16384, src.map_v, bar(B_V_FULL + vs), 64, src.row, bh);
      }
      // Readout operands, one feature piece at a time, into the freed stages.
      const uint32_t wbytes = static_cast<uint32_t>(pw) * kD * 2;
      const uint32_t slbytes = static_cast<uint32_t>(pw) * kD * 4;
      for (int pc = 0; pc < npieces && ok; ++pc) {
        if (pc == 0)
          ok = mbar_wait(bar(B_LAST_PV), 0, abort_flag, 2);
        else
          ok = mbar_wait(bar(B_READ_DONE), (pc - 1) & 1, abort_flag, 3);
        if (!ok) break;
        const __nv_bfloat16* wsrc = wq_img + (static_cast<long long>(h) * Dp + pc * pw) * kD;
        const float* slsrc = P.SL + (static_cast<long long>(bh) * P.nchunks + t) * Dp * kD +
                             static_cast<long long>(pc) * pw * kD;
        mbar_expect_tx(bar(B_TAIL_FULL), wbytes + slbytes);
        bulk_load(base + kWOff, wsrc, wbytes, bar(B_TAIL_FULL));
        bulk_load(base + kSLOff, slsrc, slbytes, bar(B_TAIL_FULL));
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ================================================= MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc(kBM, kBN, 1, false);
      const uint32_t id_pv = idesc(kBM, kD, 1, true);
      bool ok = mbar_wait(bar(B_Q_FULL), 0, abort_flag, 4);
      auto issue_s = [&](int i) -> bool {
        const int s = i & 1;
        const int ks = i % kKStages;
        if (!mbar_wait(bar(B_K_FULL + ks), (i / kKStages) & 1, abort_flag, 5)) return false;
        if (i >= 2 && !mbar_wait(bar(B_S_FREE + s), ((i - 2) >> 1) & 1, abort_flag, 6))
          return false;
        tc_fence_after();
        const uint32_t kaddr = base + kKOff + ks * kTileBytes;
        const uint32_t d = tmem + kColS0 + s * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16(d, sdesc(base + kQOff + off, 16, 1024), sdesc(kaddr + off, 16, 1024), id_qk,
                   kk > 0);
        }
        mma_commit(bar(B_S_FULL + s));
        mma_commit(bar(B_K_EMPTY + ks));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nt && ok; ++j) {
        if (j + 1 < nt) ok = issue_s(j + 1);
        if (!ok) break;
        const int s = j & 1;
        ok = mbar_wait(bar(B_P_FULL), j & 1, abort_flag, 7) &&
             mbar_wait(bar(B_V_FULL + s), (j >> 1) & 1, abort_flag, 8);
        if (!ok) break;
        tc_fence_after();
        const uint32_t vaddr = base + kVOff + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sdesc(base + kPOff + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc(vaddr + kk * 2048, 16384, 1024);
          mma_bf16(tmem + kColO, a, b, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(B_PV_DONE));
        mma_commit(bar(B_V_EMPTY + s));
        if (j == nt - 1) mma_commit(bar(B_LAST_PV));
      }
      // Linear readout, one feature piece at a time.
      const uint32_t id_phi = idesc(kBM, pw, 1, false);
      const uint32_t id_rd = idesc(kBM, kD, 2, false);
      for (int pc = 0; pc < npieces && ok; ++pc) {
        ok = mbar_wait(bar(B_TAIL_FULL), pc & 1, abort_flag, 9);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t qoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t woff = (kk >> 2) * (pw * 128) + (kk & 3) * 32;
          mma_bf16(tmem + kColS0, sdesc(base + kQOff + qoff, 16, 1024),
                   sdesc(base + kWOff + woff, 16, 1024), id_phi, kk > 0);
        }
        mma_commit(bar(B_PHI_DONE));
        ok = mbar_wait(bar(B_PHI_READY), pc & 1, abort_flag, 10);
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < pw / 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_tf32(tmem + kColAL, sdesc(base + kPhiOff + off, 16, 1024),
                   sdesc(base + kSLOff + off, 16, 1024), id_rd, (pc > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(B_READ_DONE));
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // ================================================= softmax / epilogue
    const int r = tid;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m_used = -INFINITY, m_max = -INFINITY, l = 0.f;
    bool ok = true;
    // Warp-uniform outcome, so an abort never splits a warp before the
    // warp-collective TMEM accesses.
    auto wait_all = [&](uint32_t b, uint32_t parity, uint32_t code) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, code));
    };
    for (int j = 0; j < nt && ok; ++j) {
      const int s = j & 1;
      ok = wait_all(bar(B_S_FULL + s), (j >> 1) & 1, 11);
      if (!ok) break;
      tc_fence_after();
      uint32_t xr[128];
      {
        const uint32_t sa = lane_base + kColS0 + s * 128;
        REHYAT_TMEM_LD32(sa + 0, (xr + 0));
        REHYAT_TMEM_LD32(sa + 32, (xr + 32));
        REHYAT_TMEM_LD32(sa + 64, (xr + 64));
        REHYAT_TMEM_LD32(sa + 96, (xr + 96));
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar(B_S_FREE + s));
      const int nvalid = tile_src(j).nvalid;
      if (nvalid < kBN) {  // ragged tile (warp-uniform): mask keys past the end
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i >= nvalid) xr[i] = __float_as_uint(-INFINITY);
      }
      // Row max of the raw logits as a tree (the scale is positive).
      float mx[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) mx[i] = __uint_as_float(xr[i]);
#pragma unroll
      for (int i = 16; i < 128; ++i) mx[i & 15] = fmaxf(mx[i & 15], __uint_as_float(xr[i]));
#pragma unroll
      for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
      m_max = fmaxf(m_max, mx[0] * P.scale_log2);
      float alpha = 1.f;
      const bool rescale = m_max > m_used + 8.f;
      if (rescale) {
        alpha = ex2(m_used - m_max);  // 0 on the first tile
        m_used = m_max;
      }
      // p = 2^(s * scale * log2(e) - m_used), one FFMA + one MUFU each; the
      // row sum uses 8 independent accumulators.
      const float neg_m = -m_used;
      uint32_t pk[64];
      float ls[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ls[i] = 0.f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float p0 = ex2(fmaf(__uint_as_float(xr[2 * i]), P.scale_log2, neg_m));
        const float p1 = ex2(fmaf(__uint_as_float(xr[2 * i + 1]), P.scale_log2, neg_m));
        pk[i] = pack_bf16(p0, p1);
        ls[i & 7] += p0 + p1;
      }
      l = l * alpha + (((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7])));
      if (j > 0) {
        ok = wait_all(bar(B_PV_DONE), (j - 1) & 1, 12);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
          // Bring the earlier a^S to the new reference point (warp-collective
          // TMEM access; rows that did not move scale by alpha = 1).
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t oa = lane_base + kColO + c * 32;
            REHYAT_TMEM_LD32(oa, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            REHYAT_TMEM_ST32(oa, o);
          }
          tmem_wait_st();
        }
      }
      // P row r into the K-major swizzled P tile (2 boxes of 64 keys).
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t box = c >> 3, ch = c & 7;
        const uint32_t addr = base + kPOff + box * 16384 + r * 128 + ((ch ^ (r & 7)) << 4);
        st_shared_v4(addr, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      if (nvalid < kBN) {
        // Zero the V rows past the last valid key so 0 * garbage stays 0.
        ok = wait_all(bar(B_V_FULL + s), (j >> 1) & 1, 13);
        if (!ok) break;
        if (r >= nvalid) {
          const uint32_t vrow = base + kVOff + s * kTileBytes + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            st_shared_v4(vrow + c * 16, 0, 0, 0, 0);
            st_shared_v4(vrow + 16384 + c * 16, 0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(B_P_FULL));
    }
    // Final factor: a^S, n^S relative to the true maximum c.
    const float fscale = ex2(m_used - m_max);
    float nL = 0.f;
    const float* zL = linear ? P.zL + (static_cast<long long>(bh) * P.nchunks + t) * Dp : nullptr;
    for (int pc = 0; pc < npieces && ok; ++pc) {
      ok = wait_all(bar(B_PHI_DONE), pc & 1, 14);
      if (!ok) break;
      tc_fence_after();
      for (int c = 0; c < pw / 32; ++c) {
        uint32_t v[32];
        REHYAT_TMEM_LD32(lane_base + kColS0 + c * 32, v);
        tmem_wait_ld();
        float ph[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int f = pc * pw + c * 32 + i;
          const int part = f >= (Dp >> 1);
          const float b = __ldg(P.bq + (h * 2 + part) * (Dp >> 1) + (f - part * (Dp >> 1)));
          const float psi = __uint_as_float(v[i]) + b;
          ph[i] = psi * psi;
          nL = fmaf(ph[i], __ldg(zL + f), nL);
        }
        // 32 features = one box of the K-major tf32 phi tile.
        const uint32_t rowaddr = base + kPhiOff + c * 16384 + r * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(rowaddr + ((ch ^ (r & 7)) << 4), __float_as_uint(ph[4 * ch]),
                       __float_as_uint(ph[4 * ch + 1]), __float_as_uint(ph[4 * ch + 2]),
                       __float_as_uint(ph[4 * ch + 3]));
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(B_PHI_READY));
    }
    if (ok) {
      if (npieces > 0)
        ok = wait_all(bar(B_READ_DONE), (npieces - 1) & 1, 15);
      else
        ok = wait_all(bar(B_PV_DONE), (nt - 1) & 1, 15);
    }
    if (ok) {
      tc_fence_after();
      const float nS = l * fscale;
      const float den = nS + nL;
      const long long grow = static_cast<long long>(bh) * P.rows_per_bh + row0 + r;
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32], al[32];
        REHYAT_TMEM_LD32(lane_base + kColO + c * 32, o);
        if (linear) REHYAT_TMEM_LD32(lane_base + kColAL + c * 32, al);
        tmem_wait_ld();
        if (r < nrows) {
          float yv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float aS = __uint_as_float(o[i]) * fscale;
            const float aL = linear ? __uint_as_float(al[i]) : 0.f;
            yv[i] = __fdiv_rn(aS + aL, den);
            if (P.dbg_aS) P.dbg_aS[grow * kD + c * 32 + i] = aS;
            if (P.dbg_aL) P.dbg_aL[grow * kD + c * 32 + i] = aL;
          }
          if (P.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.y) + grow * kD +
                                                  c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16(yv[8 * i], yv[8 * i + 1]),
                                  pack_bf16(yv[8 * i + 2], yv[8 * i + 3]),
                                  pack_bf16(yv[8 * i + 4], yv[8 * i + 5]),
                                  pack_bf16(yv[8 * i + 6], yv[8 * i + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(P.y) + grow * kD + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(yv[4 * i], yv[4 * i + 1], yv[4 * i + 2], yv[4 * i + 3]);
          }
        }
      }
      if (r < nrows) {
        if (P.dbg_nS) P.dbg_nS[grow] = nS;
        if (P.dbg_nL) P.dbg_nL[grow] = nL;
        if (P.dbg_c) P.dbg_c[grow] = m_max * 0.69314718055994530942f;
      }
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ===========================================================================
// Attention kernel with two query tiles per CTA (used when D' <= 128).
//
// Same computation as tc_attn_kernel, arranged so the tensor core alternates
// between two 128-row query tiles A and B of one chunk: while softmax
// warpgroup A turns S_A(j) into P_A(j), the MMA warp runs q.k^T of tile B and
// P.V of tile A, and the other way round.  P stays in TMEM (bf16, two per
// 32-bit column, over the first 64 columns of its S buffer) and feeds P.V as
// the A operand straight from TMEM, so shared memory only holds Q_A, Q_B and
// the K (3 stages) and V (2 stages) rings.  The linear readout multiplies
// phi_q(q) by 1/f (f = exp2(m_used - m_max) <= 1) and accumulates into O, so
// y = f*O / (f*n^S + n^L).
//
// Roles (320 threads): warps 0-3 softmax + epilogue of tile A, warps 4-7 of
// tile B, warp 8 TMA, warp 9 MMA and TMEM owner.
// TMEM: S_A [0,128) O_A [128,256) S_B [256,384) O_B [384,512).
// ===========================================================================
namespace a2 {
constexpr int kThreads = 320;
constexpr uint32_t kQOff = 0;                      // Q_A, Q_B
constexpr uint32_t kKOff = 65536;                  // K ring, 3 x 32 KB
constexpr uint32_t kVOff = kKOff + 3 * 32768;      // V ring, 2 x 32 KB
constexpr uint32_t kBarOff = kVOff + 2 * 32768;
constexpr uint32_t kWOff = kKOff;                  // tail: phi_q weights (<= 32 KB)
constexpr uint32_t kSLOff = kKOff + 32768;         // tail: S^L (<= 64 KB)
constexpr uint32_t kPhiOff0 = kVOff;               // tail: phi_q(Q_A)/f (<= 64 KB)
constexpr uint32_t kPhiOff1 = kQOff;               // tail: phi_q(Q_B)/f, over Q (<= 64 KB)
// fp8 softmax variant: E4M3 K tiles are 16 KB (one 128-byte box per row), so
// the K ring takes 48 KB and the E4M3 Q_A, Q_B sit in the 32 KB after it;
// the bf16 Q stays for the phi_q tail, whose operands reuse [kKOff, kVOff)
// once the last q.k^T has run.
constexpr uint32_t kK8Stage = 16384;
constexpr uint32_t kQ8Off = kKOff + 3 * kK8Stage;
enum { Q_FULL = 0, K_FULL = 1, K_EMPTY = 4, V_FULL = 7, V_EMPTY = 9, S_FULL = 11, P_FULL = 13,
       PV_DONE = 15, LAST_PV = 17, TAIL_FULL = 18, PHI_DONE = 19, PHI_READY = 20, READ_DONE = 22,
       VEC_READY = 23, XCHG = 24, LX = 26, LX_DONE = 27, READ_A = 28, NBAR = 29 };
// Row halves: each softmax thread owns 64 of a row's 128 key columns; the
// two threads of a row (warps w and w + 4, same TMEM lane quarter) trade
// their partial row maxima through TMEM column 63 (half 0) and 127 (half 1)
// of the tile's S buffer, and their partial row sums, after the key loop,
// through column 126 (a column no maximum passes through, so a slow partner
// still reading its last maximum is never overwritten).
constexpr uint32_t kXchgCol0 = 63, kXchgCol1 = 127, kLxCol = 126;
constexpr uint32_t kTmemSlot = kBarOff + 8 * NBAR;
constexpr uint32_t kAbortSlot = kTmemSlot + 4;
constexpr uint32_t kLastSlot = kAbortSlot + 4;     // split key window: this CTA merges
constexpr uint32_t kSplitSlot = kLastSlot + 4;     // (split pair slot, piece, pieces) for the tail
// Split key window (streaming step): per piece and tile, 33 float4 columns of
// 128 rows -- a^S in 32 (relative to the piece's own row maximum), then
// (maximum, row sum, 0, 0) -- so a warp's 32 rows are 512 contiguous bytes.
constexpr int kPartVec = 33;
// b_q of the head and z^L of the chunk (D' floats each), shared by both tiles.
constexpr uint32_t kVecOff = kBarOff + 256;
constexpr uint32_t kSmemBytes = kVecOff + 1024 + 1024;
}  // namespace a2

// kFp8: q.k^T from the E4M3 copies of q and k (tcgen05 kind::f8f6f4, K = 32
// per instruction); everything else as in the bf16 kernel.
template <bool kFp8>
__global__ void __launch_bounds__(a2::kThreads, 1)
    tc_attn2_kernel(const __grid_constant__ TcMaps maps, const AttnParams P,
                    const __nv_bfloat16* __restrict__ wq_img) {
  using a2::kQOff;
  using a2::kKOff;
  using a2::kVOff;
  using a2::kBarOff;
  using a2::kWOff;
  using a2::kSLOff;
  using a2::kPhiOff0;
  using a2::kPhiOff1;
  using a2::kTmemSlot;
  using a2::kAbortSlot;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + kBarOff + 8u * i; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sbase + kAbortSlot);
  // A streaming step's fold (launched next, programmatic dependent) may start
  // once every CTA of this grid has started: it touches nothing this reads.
  asm volatile("griddepcontrol.launch_dependents;");

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool step_mode = P.seen != nullptr;
  int t = blockIdx.y;
  int bh = blockIdx.z;
  int pair = blockIdx.x;      // pair of query tiles within the chunk
  int split = 0, nsplit = 1;  // piece of the key window this CTA runs
  int slot = 0;               // split pair index (partials, arrival counter)
  if (step_mode && P.ksplit > 1) {
    // Work list in dispatch order: the BH pairs that hold only tile A, then
    // kwhole two-tile pairs run whole, then the remaining two-tile pairs as
    // ksplit key pieces each.
    const int qrows = P.nq_slices * P.HW;
    const int npairs = (qrows + 2 * kBM - 1) / (2 * kBM);
    const bool light = qrows - (npairs - 1) * 2 * kBM <= kBM;
    const int nfull = npairs - (light ? 1 : 0);
    const int nl = light ? P.BH : 0;
    int L = blockIdx.x;
    t = 0;
    if (L < nl) {
      bh = L;
      pair = npairs - 1;
    } else {
      L -= nl;
      int item = L;
      if (L >= P.kwhole) {
        L -= P.kwhole;
        slot = L / P.ksplit;
        split = L % P.ksplit;
        nsplit = P.ksplit;
        item = P.kwhole + slot;
      }
      bh = item / nfull;
      pair = item % nfull;
    }
  }
  const int h = bh % P.heads;

  int q_first, q_end, na, nb, a_row0;
  if (!step_mode) {
    const int first = t * P.Tc;
    const int end = min(P.T, first + P.Tc);
    const int w = max(first - P.To, 0);
    q_first = first * P.HW;
    q_end = end * P.HW;
    a_row0 = w * P.HW;
    na = (end - w) * P.HW;
    nb = 0;
  } else {
    const long long seen = *P.seen;
    const int r_slices = static_cast<int>(seen < P.To ? seen : P.To);
    q_first = 0;
    q_end = P.nq_slices * P.HW;
    a_row0 = 0;
    na = r_slices * P.HW;
    nb = q_end;
  }
  const int row0 = q_first + pair * 2 * kBM;
  if (row0 >= q_end) return;
  const int nrows_t[2] = {min(kBM, q_end - row0), max(0, min(kBM, q_end - row0 - kBM))};
  const bool has_b = nrows_t[1] > 0;
  const int nta = (na + kBN - 1) / kBN;
  const int nt_all = nta + (nb + kBN - 1) / kBN;
  // Key tiles [j0, j0 + nt) of the window (all of it unless split; the host
  // keeps ksplit <= the chunk's own key tiles, so every piece has one).
  const int j0 = split * nt_all / nsplit;
  const int nt = (split + 1) * nt_all / nsplit - j0;
  const bool split_kv = nsplit > 1;
  const bool linear = !P.full_softmax;
  const bool phi_given = P.phi_q != nullptr;  // phi_q(q) read from P.phi_q
  const int Dp = P.Dp;
  const int npieces = Dp > 128 ? 2 : 1;       // feature pieces of the readout
  const int pw = Dp / npieces;

  auto tile_src = [&](int jl) {
    const int j = j0 + jl;
    TileSrc s;
    if (j < nta) {
      s.map_k = step_mode ? &maps.rk : &maps.k;
      s.map_v = step_mode ? &maps.rv : &maps.v;
      s.row = a_row0 + j * kBN;
      s.nvalid = min(kBN, na - j * kBN);
    } else {
      const int jb = j - nta;
      s.map_k = &maps.k;
      s.map_v = &maps.v;
      s.row = jb * kBN;
      s.nvalid = min(kBN, nb - jb * kBN);
    }
    return s;
  };

  if (tid == 0) {
    for (int i = 0; i < a2::NBAR; ++i) {
      const bool by_warpgroup = i == a2::PHI_READY || i == a2::PHI_READY + 1 || i == a2::VEC_READY;
      const bool by_all = i == a2::P_FULL || i == a2::P_FULL + 1 || i == a2::XCHG ||
                          i == a2::XCHG + 1 || i == a2::LX || i == a2::LX_DONE;
      mbar_init(bar(i), by_all ? 2 * kSoftmaxThreads : (by_warpgroup ? kSoftmaxThreads : 1));
    }
    *abort_flag = 0;
    *reinterpret_cast<volatile uint32_t*>(sbase + a2::kLastSlot) = split_kv ? 0u : 1u;
    volatile int* sp = reinterpret_cast<volatile int*>(sbase + a2::kSplitSlot);
    sp[0] = slot;
    sp[1] = split;
    sp[2] = nsplit;
    fence_barrier_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     base + kTmemSlot),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + kTmemSlot);
  // Split key window: after LX_DONE this says whether this CTA merges the
  // pieces and runs the tail (the last piece of the pair to finish).
  auto merges = [&]() { return *reinterpret_cast<volatile uint32_t*>(sbase + a2::kLastSlot) != 0; };

  if (warp == 8) {
    // ================================================= TMA producer
    if (lane == 0) {
      bool ok = true;
      mbar_expect_tx(bar(a2::Q_FULL), (kFp8 ? 6 : 4) * 16384);
      tma_load_3d(base + kQOff, &maps.q, bar(a2::Q_FULL), 0, row0, bh);
      tma_load_3d(base + kQOff + 16384, &maps.q, bar(a2::Q_FULL), 64, row0, bh);
      tma_load_3d(base + kQOff + 32768, &maps.q, bar(a2::Q_FULL), 0, row0 + kBM, bh);
      tma_load_3d(base + kQOff + 49152, &maps.q, bar(a2::Q_FULL), 64, row0 + kBM, bh);
      if (kFp8) {
        tma_load_3d(base + a2::kQ8Off, &maps.q8, bar(a2::Q_FULL), 0, row0, bh);
        tma_load_3d(base + a2::kQ8Off + 16384, &maps.q8, bar(a2::Q_FULL), 0, row0 + kBM, bh);
      }
      if (linear && phi_given) {
        // The tail reads both tiles' rows of phi_q(q) (contiguous): into L2
        // now, so those loads do not wait on DRAM at the end of the CTA.
        const int eb = P.phi_bf16 ? 2 : 4;
        const uint32_t bytes = static_cast<uint32_t>(nrows_t[0] + nrows_t[1]) * Dp * eb;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                         static_cast<const uint8_t*>(P.phi_q) +
                         (static_cast<long long>(bh) * P.rows_per_bh + row0) * Dp * eb),
                     "r"(bytes)
                     : "memory");
      }
      for (int j = 0; j < nt && ok; ++j) {
        const TileSrc src = tile_src(j);
        const int ks = j % 3;
        if (j >= 3) ok = mbar_wait(bar(a2::K_EMPTY + ks), ((j - 3) / 3) & 1, abort_flag, 1);
        if (!ok) break;
        if (kFp8) {
          const uint32_t kdst = base + kKOff + ks * a2::kK8Stage;
          mbar_expect_tx(bar(a2::K_FULL + ks), a2::kK8Stage);
          tma_load_3d(kdst, &maps.k8, bar(a2::K_FULL + ks), 0, src.row, bh);
        } else {
          const uint32_t kdst = base + kKOff + ks * 32768;
          mbar_expect_tx(bar(a2::K_FULL + ks), 32768);
          tma_load_3d(kdst, src.map_k, bar(a2::K_FULL + ks), 0, src.row, bh);
          tma_load_3d(kdst + 16384, src.map_k, bar(a2::K_FULL + ks), 64, src.row, bh);
        }
        const int vs = j & 1;
        if (j >= 2) ok = mbar_wait(bar(a2::V_EMPTY + vs), ((j - 2) >> 1) & 1, abort_flag, 26);
        if (!ok) break;
        const uint32_t vdst = base + kVOff + vs * 32768;
        mbar_expect_tx(bar(a2::V_FULL + vs), 32768);
        tma_load_3d(vdst, src.map_v, bar(a2::V_FULL + vs), 0, src.row, bh);
        tma_load_3d(vdst + 16384, src.map_v, bar(a2::V_FULL + vs), 64, src.row, bh);
      }
      // A split piece loads the tail operands only if it merges.
      if (ok && split_kv) ok = mbar_wait(bar(a2::LX_DONE), 0, abort_flag, 20) && merges();
      if (linear && ok) {
        const uint32_t wbytes = static_cast<uint32_t>(pw) * kD * 2;
        const uint32_t slbytes = static_cast<uint32_t>(pw) * kD * 4;
        // The tail operands go into the K ring as soon as the last three K
        // tiles have been consumed (their q.k^T MMAs completed), while the
        // last softmax steps and P.V still run; with two feature pieces the
        // second piece follows once both readouts of the first are done.
        for (int tt = max(0, nt - 3); tt < nt && ok; ++tt)
          ok = mbar_wait(bar(a2::K_EMPTY + tt % 3), (tt / 3) & 1, abort_flag, 2);
        for (int pc = 0; pc < npieces && ok; ++pc) {
          if (pc > 0) ok = mbar_wait(bar(a2::READ_DONE), (pc - 1) & 1, abort_flag, 2);
          if (!ok) break;
          // With phi_q(q) given there is no W_q image to load.
          mbar_expect_tx(bar(a2::TAIL_FULL), (phi_given ? 0u : wbytes) + slbytes);
          if (!phi_given)
            bulk_load(base + kWOff, wq_img + (static_cast<long long>(h) * Dp + pc * pw) * kD,
                      wbytes, bar(a2::TAIL_FULL));
          bulk_load(base + kSLOff,
                    P.SL + (static_cast<long long>(bh) * P.nchunks + t) * Dp * kD +
                        static_cast<long long>(pc) * pw * kD,
                    slbytes, bar(a2::TAIL_FULL));
        }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ================================================= MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc(kBM, kBN, 1, false);
      const uint32_t id_pv = idesc(kBM, kD, 1, true);
      const int ntiles = has_b ? 2 : 1;
      bool ok = mbar_wait(bar(a2::Q_FULL), 0, abort_flag, 4);
      auto issue_s = [&](int tile, int j) {
        if (kFp8) {
          // E4M3 rows are 128 bytes: one box, 32 elements (32 bytes) a step.
          const uint32_t kaddr = base + kKOff + (j % 3) * a2::kK8Stage;
          const uint32_t qaddr = base + a2::kQ8Off + tile * 16384;
          const uint32_t id_qk8 = idesc(kBM, kBN, 0, false);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_e4m3(tmem + tile * 256, sdesc(qaddr + kk * 32, 16, 1024),
                     sdesc(kaddr + kk * 32, 16, 1024), id_qk8, kk > 0);
        } else {
          const uint32_t kaddr = base + kKOff + (j % 3) * 32768;
          const uint32_t qaddr = base + kQOff + tile * 32768;
          mma8_ss_kmajor(tmem + tile * 256, sdesc(qaddr, 16, 1024), sdesc(kaddr, 16, 1024), id_qk,
                         0u);
        }
        mma_commit(bar(a2::S_FULL + tile));
      };
      auto issue_pv = [&](int tile, int j) {
        const uint32_t vaddr = base + kVOff + (j & 1) * 32768;
        mma8_ts_mn(tmem + tile * 256 + 128, tmem + tile * 256, sdesc(vaddr, 16384, 1024), id_pv,
                   j > 0 ? 1u : 0u);
        mma_commit(bar(a2::PV_DONE + tile));
      };
      if (ok) ok = mbar_wait(bar(a2::K_FULL), 0, abort_flag, 5);
      if (ok) {
        tc_fence_after();
        for (int tile = 0; tile < ntiles; ++tile) issue_s(tile, 0);
        mma_commit(bar(a2::K_EMPTY));
      }
      for (int j = 0; j < nt && ok; ++j) {
        const int vs = j & 1;
        const bool more = j + 1 < nt;
        ok = mbar_wait(bar(a2::V_FULL + vs), (j >> 1) & 1, abort_flag, 8);
        if (ok && more)
          ok = mbar_wait(bar(a2::K_FULL + (j + 1) % 3), ((j + 1) / 3) & 1, abort_flag, 5);
        for (int tile = 0; tile < ntiles && ok; ++tile) {
          ok = mbar_wait(bar(a2::P_FULL + tile), j & 1, abort_flag, 7);
          if (!ok) break;
          tc_fence_after();
          issue_pv(tile, j);                  // reads P(j) from this tile's S columns
          if (more) issue_s(tile, j + 1);     // then overwrites them (in-order pipe)
        }
        if (!ok) break;
        mma_commit(bar(a2::V_EMPTY + vs));
        if (more) mma_commit(bar(a2::K_EMPTY + (j + 1) % 3));
        if (j == nt - 1) mma_commit(bar(a2::LAST_PV));
      }
      if (ok && split_kv) ok = mbar_wait(bar(a2::LX_DONE), 0, abort_flag, 20) && merges();
      // Linear readout, one feature piece of pw <= 128 at a time.
      for (int pc = 0; linear && ok && pc < npieces; ++pc) {
        ok = mbar_wait(bar(a2::TAIL_FULL), pc & 1, abort_flag, 9);
        // The phi_q product overwrites S: the softmax warps have traded
        // their row sums through it first.
        if (ok && pc == 0 && !phi_given) ok = mbar_wait(bar(a2::LX_DONE), 0, abort_flag, 18);
        if (!ok) break;
        tc_fence_after();
        if (!phi_given) {
          const uint32_t id_phi = idesc(kBM, pw, 1, false);
          for (int tile = 0; tile < ntiles; ++tile)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t qoff = tile * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32;
              const uint32_t woff = (kk >> 2) * (pw * 128) + (kk & 3) * 32;
              mma_bf16(tmem + tile * 256, sdesc(base + kQOff + qoff, 16, 1024),
                       sdesc(base + kWOff + woff, 16, 1024), id_phi, kk > 0);
            }
          mma_commit(bar(a2::PHI_DONE));
        }
        const uint32_t id_rd = idesc(kBM, kD, 2, false);
        for (int tile = 0; tile < ntiles && ok; ++tile) {
          ok = mbar_wait(bar(a2::PHI_READY + tile), pc & 1, abort_flag, 10);
          if (!ok) break;
          tc_fence_after();
          // One piece: tile A's phi_q sits in the V ring, tile B's over Q.
          // Two pieces: Q is read again for the second piece, so both tiles
          // stage in the V ring, tile B after tile A's readout (READ_A).
          const uint32_t phi = base + ((tile && npieces == 1) ? kPhiOff1 : kPhiOff0);
          for (int kk = 0; kk < pw / 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_tf32(tmem + tile * 256 + 128, sdesc(phi + off, 16, 1024),
                     sdesc(base + kSLOff + off, 16, 1024), id_rd, 1u);
          }
          if (tile == 0 && npieces > 1) mma_commit(bar(a2::READ_A));
        }
        if (ok) mma_commit(bar(a2::READ_DONE));
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ================================================= softmax / epilogue
    // Key loop: all eight warps work on each query tile in turn (tile A,
    // then tile B, per key step), two threads per row: warp w handles key
    // columns [64 hf, 64 hf + 64) of rows 32 (w & 3) .. + 31, hf = w >> 2.
    // Both threads of a row take the same reference point (the partial
    // maxima are traded through TMEM), so their P values add up in one P.V.
    // Tail: warps 0-3 finish tile A, warps 4-7 tile B (as one warpgroup each).
    const int hf = warp >> 2;
    const int r = tid & 127;                 // row within a tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int ntiles = has_b ? 2 : 1;
    float m_used2[2] = {-INFINITY, -INFINITY}, m_max2[2] = {-INFINITY, -INFINITY};
    float l2[2] = {0.f, 0.f};                // this thread's half of each row sum
    bool ok = true;
    auto wait_all = [&](uint32_t b, uint32_t parity, uint32_t code) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, code));
    };
    float* vec = reinterpret_cast<float*>(sbase + a2::kVecOff);  // [b_q (D') | z^L (D')]
    if (linear && hf == 0) {
      // Warps 0-3 stage b_q and z^L for the tail while they wait for the
      // first scores (b_q of head h is h's D' consecutive values; one
      // feature piece only, D' <= 128).
      if (r < Dp && npieces == 1) {
        vec[r] = phi_given ? 0.f : __ldg(P.bq + h * Dp + r);
        vec[Dp + r] = __ldg(P.zL + (static_cast<long long>(bh) * P.nchunks + t) * Dp + r);
      }
      mbar_arrive(bar(a2::VEC_READY));
    }
    const uint64_t scale2 = f2_pack(P.scale_log2, P.scale_log2);
    const uint32_t my_xcol = hf ? a2::kXchgCol1 : a2::kXchgCol0;
    const uint32_t other_xcol = hf ? a2::kXchgCol0 : a2::kXchgCol1;
    for (int j = 0; j < nt && ok; ++j) {
      const int nvalid = tile_src(j).nvalid;
      const bool ragged = nvalid < kBN;  // warp-uniform: keys past the end
      for (int tile = 0; tile < ntiles && ok; ++tile) {
        const uint32_t s_col = tile * 256, o_col = s_col + 128;
        // S_FULL(j) also covers this tile's P.V of step j-1 (issued earlier).
        ok = wait_all(bar(a2::S_FULL + tile), j & 1, 11);
        if (!ok) break;
        tc_fence_after();
        uint32_t x[64];
        REHYAT_TMEM_LD32(lane_base + s_col + 64 * hf, x);
        REHYAT_TMEM_LD32(lane_base + s_col + 64 * hf + 32, (x + 32));
        tmem_wait_ld();
        if (ragged) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (64 * hf + i >= nvalid) x[i] = __float_as_uint(-INFINITY);
        }
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          mx[i] = fmax3(fmax3(__uint_as_float(x[i]), __uint_as_float(x[i + 8]),
                              __uint_as_float(x[i + 16])),
                        fmax3(__uint_as_float(x[i + 24]), __uint_as_float(x[i + 32]),
                              __uint_as_float(x[i + 40])),
                        fmaxf(__uint_as_float(x[i + 48]), __uint_as_float(x[i + 56])));
        float pm = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                         fmaxf(mx[6], mx[7]));
        // Trade the partial maxima: each thread writes its own into a column
        // of its half of S (already in registers), reads its partner's.
        tmem_st1(lane_base + s_col + my_xcol, __float_as_uint(pm));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(a2::XCHG + tile));
        ok = wait_all(bar(a2::XCHG + tile), j & 1, 16);
        if (!ok) break;
        tc_fence_after();
        pm = fmaxf(pm, __uint_as_float(tmem_ld1(lane_base + s_col + other_xcol)));
        float& m_max = m_max2[tile];
        float& m_used = m_used2[tile];
        m_max = fmaxf(m_max, pm * P.scale_log2);
        float alpha = 1.f;
        // The reference point moves only when the maximum passes it by more
        // than 16 (log2 units): p <= 2^16 and a row's sum <= 2^16 per key stay
        // far inside fp32 and bf16 range, and the final factor
        // 2^(m_used - m_max) makes the result exact with respect to c.
        const bool rescale = m_max > m_used + 16.f;
        if (rescale) {
          alpha = ex2(m_used - m_max);  // 0 on the first tile
          m_used = m_max;
        }
        // p = 2^(s * scale * log2(e) - m_used) on packed fp32 pairs (MUFU
        // ex2); P (bf16 pairs) of this half goes to S columns
        // [32 hf, 32 hf + 32): half 1 overwrites column 63 only after it
        // has read it.
        const uint64_t negm2 = f2_pack(-m_used, -m_used);
        uint64_t ls2[4] = {0, 0, 0, 0};
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(x[2 * i]),
                                             __uint_as_float(x[2 * i + 1])),
                                     scale2, negm2);
          float a0, a1;
          f2_unpack(x2, a0, a1);
          const uint64_t p2 = f2_pack(ex2(a0), ex2(a1));
          float p0, p1;
          f2_unpack(p2, p0, p1);
          pk[i] = pack_bf16(p0, p1);
          ls2[i & 3] = f2_add(ls2[i & 3], p2);
        }
        REHYAT_TMEM_ST32(lane_base + s_col + 32 * hf, pk);
        float ls[4];
        f2_unpack(f2_add(ls2[0], ls2[1]), ls[0], ls[1]);
        f2_unpack(f2_add(ls2[2], ls2[3]), ls[2], ls[3]);
        // This tile's P.V of step j-1 is complete (covered by S_FULL(j)):
        // bring this half's columns of the earlier a^S to the new reference
        // point.  Warp-collective; rows that did not move use alpha = 1.
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            REHYAT_TMEM_LD32(lane_base + o_col + 64 * hf + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            REHYAT_TMEM_ST32(lane_base + o_col + 64 * hf + c * 32, o);
          }
        }
        tmem_wait_st();
        l2[tile] = l2[tile] * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
        if (tile == 0 && ragged) {
          // Zero the V rows past the last valid key (shared by both tiles;
          // tile B's P.V is issued after tile A's P_FULL): half hf clears
          // box hf (64 columns) of row r.
          ok = wait_all(bar(a2::V_FULL + (j & 1)), (j >> 1) & 1, 13);
          if (!ok) break;
          if (r >= nvalid) {
            const uint32_t vrow = base + kVOff + (j & 1) * 32768 + hf * 16384 + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) st_shared_v4(vrow + c * 16, 0, 0, 0, 0);
          }
          fence_proxy_async();
        }
        tc_fence_before();
        mbar_arrive(bar(a2::P_FULL + tile));
      }
    }
    // Row sums: the tail of tile A runs on half 0, that of tile B on half 1;
    // each needs the other half's part, passed through column 126 of the
    // tile's S buffer (free now: P uses columns [0, 64)).  The MMA warp
    // issues the phi_q product, which overwrites S, only after LX_DONE.
    if (ok) {
      const int give = 1 - hf;  // the tile whose tail the other half runs
      if (give < ntiles) {
        tmem_st1(lane_base + give * 256 + a2::kLxCol, __float_as_uint(l2[give]));
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(a2::LX));
      ok = wait_all(bar(a2::LX), 0, 17);
    }
    const int tile = hf;
    if (ok && tile < ntiles) {
      tc_fence_after();
      l2[tile] += __uint_as_float(tmem_ld1(lane_base + tile * 256 + a2::kLxCol));
    }
    bool run_tail = true;
    if (split_kv) {
      const volatile int* sp = reinterpret_cast<const volatile int*>(sbase + a2::kSplitSlot);
      const int slot = sp[0], split = sp[1], nsplit = sp[2];
      // Split key window (both tiles present): every piece leaves its a^S,
      // row maximum and row sum in the partials; the last piece of the pair
      // to arrive folds the others into its own TMEM accumulator and runs
      // the tail.  Nothing waits on another CTA.
      const int nrows = nrows_t[tile];
      float4* part = reinterpret_cast<float4*>(P.part);
      auto part_at = [&](int piece, int cc) {
        return part + ((static_cast<long long>(slot * nsplit + piece) * 2 + tile) * a2::kPartVec +
                       cc) * kBM + r;
      };
      ok = wait_all(bar(a2::LAST_PV), 0, 19);
      if (ok) {
        tc_fence_after();
        const float fs = ex2(m_used2[tile] - m_max2[tile]);
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          REHYAT_TMEM_LD32(lane_base + tile * 256 + 128 + c * 32, o);
          tmem_wait_ld();
          if (r < nrows)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *part_at(split, c * 8 + i) =
                  make_float4(__uint_as_float(o[4 * i]) * fs, __uint_as_float(o[4 * i + 1]) * fs,
                              __uint_as_float(o[4 * i + 2]) * fs, __uint_as_float(o[4 * i + 3]) * fs);
        }
        if (r < nrows) *part_at(split, 32) = make_float4(m_max2[tile], l2[tile] * fs, 0.f, 0.f);
      }
      __threadfence();
      asm volatile("bar.sync 3, %0;" ::"r"(2 * kSoftmaxThreads) : "memory");
      volatile uint32_t* last_slot = reinterpret_cast<volatile uint32_t*>(sbase + a2::kLastSlot);
      if (tid == 0) {
        unsigned* cnt = P.part_cnt + slot;
        const bool last = atomicAdd(cnt, 1u) == static_cast<unsigned>(nsplit - 1);
        if (last) atomicExch(cnt, 0u);  // ready for the next launch
        __threadfence();
        *last_slot = last ? 1u : 0u;
      }
      asm volatile("bar.sync 3, %0;" ::"r"(2 * kSoftmaxThreads) : "memory");
      run_tail = *last_slot != 0;
      if (ok && run_tail) {  // warp-uniform: the TMEM stores are collective
        // Every piece, this CTA's own included, is read back from the
        // partials and summed in piece order, so y does not depend on which
        // piece arrived last.
        const bool valid = r < nrows;
        float mp[4], w[4];
        float mx = -INFINITY, l = 0.f;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          const float4 ml = valid && pc < nsplit ? __ldcg(part_at(pc, 32))
                                                 : make_float4(-INFINITY, 0.f, 0.f, 0.f);
          mp[pc] = ml.x;
          w[pc] = ml.y;  // row sum for now
          mx = fmaxf(mx, ml.x);
        }
        if (!valid) mx = 0.f;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {
          const float sum = w[pc];
          w[pc] = valid && pc < nsplit ? ex2(mp[pc] - mx) : 0.f;
          l = fmaf(sum, w[pc], l);
        }
        for (int c = 0; c < 4; ++c) {
          float o[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
#pragma unroll
          for (int pc = 0; pc < 4; ++pc) {
            if (!(valid && pc < nsplit)) continue;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 v4 = __ldcg(part_at(pc, c * 8 + i));
              o[4 * i] = fmaf(v4.x, w[pc], o[4 * i]);
              o[4 * i + 1] = fmaf(v4.y, w[pc], o[4 * i + 1]);
              o[4 * i + 2] = fmaf(v4.z, w[pc], o[4 * i + 2]);
              o[4 * i + 3] = fmaf(v4.w, w[pc], o[4 * i + 3]);
            }
          }
          uint32_t ob[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) ob[i] = __float_as_uint(o[i]);
          REHYAT_TMEM_ST32(lane_base + tile * 256 + 128 + c * 32, ob);
        }
        tmem_wait_st();
        m_used2[tile] = mx;
        m_max2[tile] = mx;
        l2[tile] = l;
      }
    }
    tc_fence_before();
    mbar_arrive(bar(a2::LX_DONE));
    if (tile >= ntiles || !run_tail) {
      // Tile B is empty (warps 4-7 have no tail), or another piece of this
      // pair merges and writes y.
    } else {
    const uint32_t s_col = tile * 256, o_col = s_col + 128;
    const int nrows = nrows_t[tile];
    const float m_used = m_used2[tile], m_max = m_max2[tile], l = l2[tile];
    const float fscale = ex2(m_used - m_max);
    const long long grow = static_cast<long long>(bh) * P.rows_per_bh + row0 + tile * kBM + r;
    const bool dbg_split = P.dbg_aS != nullptr || P.dbg_aL != nullptr;
    float nL = 0.f;
    if (ok && linear) {
      if (dbg_split) {
        // a^S before the readout adds into O (debug export only).
        ok = wait_all(bar(a2::LAST_PV), 0, 14);
        if (ok) {
          tc_fence_after();
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            REHYAT_TMEM_LD32(lane_base + o_col + c * 32, o);
            tmem_wait_ld();
            if (r < nrows && P.dbg_aS)
              for (int i = 0; i < 32; ++i)
                P.dbg_aS[grow * kD + c * 32 + i] = __uint_as_float(o[i]) * fscale;
            if (r < nrows && P.dbg_aL)  // a^S for now; replaced by a^L below
              for (int i = 0; i < 32; ++i)
                P.dbg_aL[grow * kD + c * 32 + i] = __uint_as_float(o[i]) * fscale;
          }
        }
      }
      // phi_q(q) of each feature piece is staged as a tf32 operand.  One
      // piece: tile A in the V ring, tile B over Q; the closed form waits for
      // the phi MMAs (which read Q), phi_q given for the last P.V.  Two
      // pieces: both tiles in the V ring (Q is read again for the second
      // piece), tile B once tile A's readout of the piece has run (READ_A),
      // tile A's second piece once the first piece's readouts have run; b_q
      // and z^L come straight from global memory (the staged copy in shared
      // memory holds one piece).
      const float inv_f = 1.0f / fscale;
      const uint32_t phi = base + ((tile && npieces == 1) ? kPhiOff1 : kPhiOff0);
      for (int pc = 0; ok && pc < npieces; ++pc) {
        if (npieces == 1) {
          ok = wait_all(bar(a2::VEC_READY), 0, 14) &&
               wait_all(bar(phi_given ? a2::LAST_PV : a2::PHI_DONE), 0, 14);
        } else {
          ok = wait_all(bar(phi_given ? a2::LAST_PV : a2::PHI_DONE), phi_given ? 0 : (pc & 1), 14);
          if (ok && tile == 1) ok = wait_all(bar(a2::READ_A), pc & 1, 14);
          if (ok && tile == 0 && pc > 0) ok = wait_all(bar(a2::READ_DONE), (pc - 1) & 1, 14);
        }
        if (!ok) break;
        tc_fence_after();
        const int f0 = pc * pw;
        const float* zsrc = P.zL + (static_cast<long long>(bh) * P.nchunks + t) * Dp + f0;
        if (phi_given) {
          // Each warp stages its 32 rows' phi_q(q) four rows per load
          // instruction (eight lanes read a row's 32-feature chunk, 128
          // contiguous bytes): row-per-thread fp32 loads would thrash the
          // small L1 beside this kernel's shared memory.  The row's thread
          // keeps its n^L (the eight lanes' parts summed, then passed on).
          const int q4 = lane & 7, rsub = lane >> 3;
          const long long gtile = static_cast<long long>(bh) * P.rows_per_bh + row0 + tile * kBM;
          for (int c = 0; c < pw / 32; ++c) {
            const int col = c * 32 + 4 * q4;
            float z4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              z4[e] = npieces == 1 ? vec[Dp + col + e] : __ldg(zsrc + col + e);
            // One row group of four: its values (already loaded), n^L parts
            // and the tf32 staging.
            auto stage4 = [&](int it, float4 g4) {
              const int rr = 32 * (warp & 3) + 4 * it + rsub;  // row within the tile
              const float inv_r = __shfl_sync(0xffffffffu, inv_f, 4 * it + rsub);
              float part = g4.x * z4[0] + g4.y * z4[1] + g4.z * z4[2] + g4.w * z4[3];
              part += __shfl_xor_sync(0xffffffffu, part, 4);
              part += __shfl_xor_sync(0xffffffffu, part, 2);
              part += __shfl_xor_sync(0xffffffffu, part, 1);
              const float mine = __shfl_sync(0xffffffffu, part, 8 * (lane & 3));
              if ((lane >> 2) == it) nL += mine;
              st_shared_v4(phi + c * 16384 + rr * 128 + ((q4 ^ (rr & 7)) << 4),
                           __float_as_uint(g4.x * inv_r), __float_as_uint(g4.y * inv_r),
                           __float_as_uint(g4.z * inv_r), __float_as_uint(g4.w * inv_r));
            };
            const int rbase = 32 * (warp & 3) + rsub;
            if (P.phi_bf16) {
              const __nv_bfloat16* src =
                  static_cast<const __nv_bfloat16*>(P.phi_q) + (gtile + rbase) * Dp + f0 + col;
              uint2 u[8];
#pragma unroll
              for (int it = 0; it < 8; ++it)
                u[it] = rbase + 4 * it < nrows
                            ? __ldg(reinterpret_cast<const uint2*>(src + 4LL * it * Dp))
                            : make_uint2(0u, 0u);
#pragma unroll
              for (int it = 0; it < 8; ++it)
                stage4(it, make_float4(__uint_as_float(u[it].x << 16),
                                       __uint_as_float(u[it].x & 0xFFFF0000u),
                                       __uint_as_float(u[it].y << 16),
                                       __uint_as_float(u[it].y & 0xFFFF0000u)));
            } else {
              const float* src = static_cast<const float*>(P.phi_q) + (gtile + rbase) * Dp + f0 + col;
              float4 g[8];
#pragma unroll
              for (int it = 0; it < 8; ++it)
                g[it] = rbase + 4 * it < nrows
                            ? __ldg(reinterpret_cast<const float4*>(src + 4LL * it * Dp))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int it = 0; it < 8; ++it) stage4(it, g[it]);
            }
          }
        } else {
          for (int c = 0; c < pw / 32; ++c) {
            float ph[32];
            uint32_t v[32];
            REHYAT_TMEM_LD32(lane_base + s_col + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float b = npieces == 1 ? vec[c * 32 + i] : __ldg(P.bq + h * Dp + f0 + c * 32 + i);
              const float psi = __uint_as_float(v[i]) + b;
              ph[i] = psi * psi;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float z = npieces == 1 ? vec[Dp + c * 32 + i] : __ldg(zsrc + c * 32 + i);
              nL = fmaf(ph[i], z, nL);
              ph[i] *= inv_f;
            }
            const uint32_t rowaddr = phi + c * 16384 + r * 128;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              st_shared_v4(rowaddr + ((ch ^ (r & 7)) << 4), __float_as_uint(ph[4 * ch]),
                           __float_as_uint(ph[4 * ch + 1]), __float_as_uint(ph[4 * ch + 2]),
                           __float_as_uint(ph[4 * ch + 3]));
          }
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bar(a2::PHI_READY + tile));
      }
      if (ok) ok = wait_all(bar(a2::READ_DONE), (npieces - 1) & 1, 15);
    } else if (ok) {
      ok = wait_all(bar(a2::LAST_PV), 0, 15);
    }
    if (ok) {
      tc_fence_after();
      const float nS = l * fscale;
      const float den = nS + nL;
      // A signed phi (given) can drive n^L towards -n^S: count the rows, the
      // output stays as the formula gives it.
      if (phi_given && r < nrows && !(den >= ldexpf(nS, -10))) atomicAdd(&rehyat_tc_den_rows, 1ull);
      // y = f * O / den: one IEEE division per row, then a product per value.
      const float ysc = __fdiv_rn(fscale, den);
      const bool dbg_num = P.dbg_aL != nullptr || (P.dbg_aS != nullptr && !linear);
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        REHYAT_TMEM_LD32(lane_base + o_col + c * 32, o);
        tmem_wait_ld();
        if (r < nrows) {
          float yv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) yv[i] = __uint_as_float(o[i]) * ysc;
          if (dbg_num) {
            for (int i = 0; i < 32; ++i) {
              const float num = __uint_as_float(o[i]) * fscale;  // a^S + a^L
              if (P.dbg_aL) {
                float* d = P.dbg_aL + grow * kD + c * 32 + i;
                *d = linear ? num - *d : 0.f;
              }
              if (P.dbg_aS && !linear) P.dbg_aS[grow * kD + c * 32 + i] = num;
            }
          }
          if (P.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(P.y) + grow * kD +
                                                  c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16(yv[8 * i], yv[8 * i + 1]),
                                  pack_bf16(yv[8 * i + 2], yv[8 * i + 3]),
                                  pack_bf16(yv[8 * i + 4], yv[8 * i + 5]),
                                  pack_bf16(yv[8 * i + 6], yv[8 * i + 7]));
          } else {
            // fp32 rows go through shared memory (the K ring is free now:
            // tile A at kKOff, tile B 64 KB above), 16-byte chunk cc of row
            // r at position cc ^ (r & 7) so neither side has bank conflicts.
            const uint32_t srow = base + kKOff + tile * 65536 + r * 512;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t cc = c * 8 + i;
              st_shared_v4(srow + ((cc ^ (r & 7)) << 4), __float_as_uint(yv[4 * i]),
                           __float_as_uint(yv[4 * i + 1]), __float_as_uint(yv[4 * i + 2]),
                           __float_as_uint(yv[4 * i + 3]));
            }
          }
        }
      }
      if (r < nrows) {
        if (P.dbg_nS) P.dbg_nS[grow] = nS;
        if (P.dbg_nL) P.dbg_nL[grow] = nL;
        if (P.dbg_c) P.dbg_c[grow] = m_max * 0.69314718055994530942f;
      }
    }
    // Every thread of this warpgroup gets here (aborted or not), so the
    // named barrier cannot hang.  Then each warp writes whole 512-byte rows
    // of the staged fp32 output: lane l stores chunk l (coalesced).
    asm volatile("bar.sync %0, %1;" ::"r"(1 + tile), "r"(kSoftmaxThreads) : "memory");
    if (ok && !P.out_bf16) {
      const long long grow0 = static_cast<long long>(bh) * P.rows_per_bh + row0 + tile * kBM;
      for (int rr = warp & 3; rr < nrows; rr += 4) {
        const uint32_t src = base + kKOff + tile * 65536 + rr * 512 + ((lane ^ (rr & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                     : "r"(src));
        reinterpret_cast<uint4*>(static_cast<float*>(P.y) + (grow0 + rr) * kD)[lane] =
            make_uint4(a0, a1, a2, a3);
      }
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ===========================================================================
// Per-slice linear state on tensor cores (the linear branch's sums of
// phi_k(k) v^T and of phi_k(k), "Key designs 1 and 4"):
//   P_s = phi_k(K_s)^T V_s  ([D'][D] fp32),  z_s = sum_j phi_k(k_j)  ([D']),
// for every slice (full forward) or for the slices leaving the softmax window
// in a streaming step.  Persistent CTAs each stream a contiguous run of
// items through one K/V pipeline that does not drain between slices.  The
// feature map is
// computed transposed, psi^T = W_k^T K^T (TMEM lane = feature, column =
// token), so each converter thread owns one feature: it squares psi + b in
// place, rounds to bf16 and leaves phi^T in TMEM as the A operand of
// P += phi^T V (the TMEM-A form), and it sums z = sum_t phi itself.
//   warps 0-3  convert (thread = feature), z;
//   warps 4-7  epilogue: drain the finished slice's P from TMEM;
//   warp 8     TMA of K tiles (and the W_k piece when (head, half) changes);
//   warp 11    TMA of V tiles;
//   warp 9     MMA psi^T = W_k^T K^T, and TMEM owner;
//   warp 10    MMA P += phi^T V (a second issuer, so the two streams' waits
//              and issue overheads overlap in front of one tensor pipe).
// TMEM: psi^T buffers [0,128) [128,256) and phi^T buffers [256,320) [320,384)
// (alternating per token tile; phi^T is bf16 pairs, so psi^T of the tile
// after next can be written as soon as the converter has read this one),
// one P accumulator [384,512) (the epilogue drains it while the next item's
// first tile is converted).
// D' in {64, 128, 256}: with D' = 256 an item is one 128-feature half of a
// slice (items run over (b*h, half, slice), so W_k changes only at half or
// head boundaries); with D' = 64 the upper 64 W_k rows stay zero.
// ===========================================================================
// Tensor maps of the state kernel: k, v of the chunk (or of all slices) and
// the ring's k, v (streaming; equal to k, v otherwise).
struct StMaps {
  CUtensorMap k, v, rk, rv;
  CUtensorMap phik;  // phi_k(k) given: fp32 [BH][N][Dp], boxes of 32 features x 128 rows
};

namespace sp {
constexpr int kThreads = 384;
constexpr int kStages = 3;             // K and V ring depth
constexpr uint32_t kKOff = 0;          // K ring, 3 x 32 KB
constexpr uint32_t kVOff = 98304;      // V ring, 3 x 32 KB
constexpr uint32_t kWOff = 196608;     // W_k piece, 2 boxes x 128 rows x 128 B
constexpr uint32_t kBarOff = 229376;
enum { K_FULL = 0, K_EMPTY = 3, V_FULL = 6, V_EMPTY = 9, PSI_FULL = 12, PSI_FREE = 14,
       PHI_FULL = 16, PHI_FREE = 18, ACC_DONE = 20, P_FREE = 21, W_FULL = 22, W_FREE = 23,
       NBAR = 24 };
constexpr uint32_t kTmemSlot = kBarOff + 8 * NBAR;
constexpr uint32_t kAbortSlot = kTmemSlot + 4;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
// TMEM: psi^T fp32 [0,128) [128,256), phi^T bf16 pairs [256,320) [320,384)
// (each alternating per token tile), P accumulator [384,512).
constexpr uint32_t kColPsi = 0, kColPhi = 256, kColP = 384;
// phi_k(k) given: the 16 KB box b (128 tokens x 128 bytes of features,
// token-major) of stage s.  fp32 tiles (four boxes for 128 features) use two
// stages over the K ring and the W_k area; bf16 tiles (two boxes) three
// stages in the K ring, like K tiles.
constexpr int phi_stages(bool bf16) { return bf16 ? 3 : 2; }
__host__ __device__ constexpr uint32_t phi_box(int s, int b, bool bf16) {
  return bf16 ? kKOff + s * 32768 + b * 16384
              : (s == 0 ? kKOff + b * 16384
                        : (b < 2 ? kKOff + 65536 + b * 16384 : kWOff + (b - 2) * 16384));
}

// Walk over a CTA's run of items i = q * T + slice, q = bh * halves + half,
// with a division only when one (bh, half) run of slices ends.
// Items past `active` slices of a run (streaming: slots beyond the number of
// slices leaving the window this step) are skipped by every role alike.
struct ItemWalk {
  int T, halves, heads, pw, active;
  int slice = 0, q = 0;
  int wkey = 0;  // (head, half) key of the W_k piece the item needs
  __device__ int bh() const { return halves == 2 ? q >> 1 : q; }
  __device__ int half() const { return q - bh() * halves; }
  __device__ int key() const { return (bh() % heads) * halves + half(); }
  __device__ bool on() const { return slice < active; }
  // Output slot of the item: (bh, slice) with `nslots` slots per (b,h).
  __device__ long long out_index(int nslots) const {
    return static_cast<long long>(bh()) * nslots + slice;
  }
  __device__ void start(int item) {
    slice = item % T;
    q = item / T;
    wkey = key();
  }
  __device__ void next() {
    if (++slice == T) {
      slice = 0;
      ++q;
      wkey = key();
    }
  }
};
}  // namespace sp

// kPhiGiven: phi_k(k) is read from P.phi_k (full forward) instead of being
// computed from K and W_k, in fp32 or (kPhiBf16) bf16 (separate
// instantiations, so no path carries branches for the others).
template <bool kPhiGiven, bool kPhiBf16 = false>
__global__ void __launch_bounds__(sp::kThreads, 1)
    tc_state_persistent_kernel(const __grid_constant__ StMaps maps, const PartialParams P,
                               const __nv_bfloat16* __restrict__ wk_img, int items_per_cta) {
  // Local names shadow the attention kernel's constants of the same names.
  constexpr int kS = sp::kStages;
  constexpr uint32_t kKOff = sp::kKOff, kVOff = sp::kVOff, kWOff = sp::kWOff;
  constexpr uint32_t kColPsi = sp::kColPsi, kColPhi = sp::kColPhi, kColP = sp::kColP;
  using sp::K_FULL;
  using sp::K_EMPTY;
  using sp::V_FULL;
  using sp::V_EMPTY;
  using sp::PSI_FULL;
  using sp::PSI_FREE;
  using sp::PHI_FULL;
  using sp::PHI_FREE;
  using sp::ACC_DONE;
  using sp::P_FREE;
  using sp::W_FULL;
  using sp::W_FREE;
  using sp::NBAR;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + sp::kBarOff + 8u * i; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sbase + sp::kAbortSlot);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Dp = P.Dp, HW = P.HW;
  const int pw = Dp < 128 ? Dp : 128;  // features per item
  const int halves = Dp / pw;
  // Full forward: items (bh, half, slice) over all slices.  Streaming fold:
  // items (bh, half, slot) over the chunk's slots, of which the first
  // `leave` hold slices leaving the window (slot i = global slice
  // seen - min(seen, T_o) + i, in the ring if already seen, else in the chunk).
  const bool step = P.seen != nullptr;
  constexpr bool phi_given = kPhiGiven;
  constexpr bool phi_bf16 = kPhiBf16;
  const int T = step ? P.nq_slices : P.nslots;
  const long long seen0 = step ? *P.seen : 0;
  const long long rseen = seen0 < P.To ? seen0 : P.To;
  int leave = T;
  if (step) {
    const long long after = seen0 + P.nq_slices;
    leave = static_cast<int>(rseen + P.nq_slices - (after < P.To ? after : P.To));
  }
  const int total = P.BH * halves * T;
  const int it0 = blockIdx.x * items_per_cta;
  const int it1 = min(total, it0 + items_per_cta);
  // Launched as a programmatic dependent of the attention kernel of the same
  // streaming step, this grid overlaps it; waiting here before exit makes
  // this grid's completion imply the attention kernel's (no-op otherwise).
  auto dependency_wait = [] { asm volatile("griddepcontrol.wait;" ::: "memory"); };
  asm volatile("griddepcontrol.launch_dependents;");  // the chunk scan waits on the device
  if (it0 >= it1) {
    dependency_wait();
    return;
  }
  const int nitems = it1 - it0;
  const int nt = (HW + 127) / 128;
  int nactive = 0;
  {
    sp::ItemWalk w{T, halves, P.heads, pw, leave};
    w.start(it0);
    for (int il = 0; il < nitems; ++il, w.next()) nactive += w.on();
  }
  const int TT = nactive * nt;  // token tiles of this CTA

  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) {
      const bool by_group = i == PSI_FREE || i == PSI_FREE + 1 || i == PHI_FULL ||
                            i == PHI_FULL + 1 || i == P_FREE ||
                            (phi_given && (i == K_EMPTY || i == K_EMPTY + 1 || i == K_EMPTY + 2));
      mbar_init(bar(i), by_group ? 128 : 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (pw < 128) {
    // Rows pw..127 of both W_k boxes stay zero (the bulk loads fill rows
    // 0..pw-1), so psi^T is 0 on the unused lanes.
    const int per_box = (128 - pw) * 8;  // 16-byte chunks
    for (int c = tid; c < 2 * per_box; c += sp::kThreads)
      st_shared_v4(base + kWOff + (c / per_box) * 16384 + pw * 128 + (c % per_box) * 16, 0, 0,
                   0, 0);
  }
  fence_proxy_async();
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     base + sp::kTmemSlot),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + sp::kTmemSlot);

  if (warp == 8 || warp == 11) {
    // ================================================= TMA producers
    // warp 8 loads K tiles (and the W_k piece), warp 11 V tiles, so K runs
    // ahead on its own ring (psi^T) while V waits for phi^T V to free stages.
    if (lane == 0 && warp == 8 && phi_given) {
      // phi_k(k) given: its tiles (pw features x 128 tokens, boxes of 128
      // bytes of features: 32 fp32 or 64 bf16) into two stages of the space K
      // and W_k leave unused, so the converters read them from shared memory.
      bool ok = true;
      sp::ItemWalk w{T, halves, P.heads, pw, leave};
      w.start(it0);
      int gt = 0;
      constexpr bool bf = phi_bf16;
      constexpr int fpb = bf ? 64 : 32;  // features per box
      constexpr int nst = sp::phi_stages(bf);
      const uint32_t tile_bytes = static_cast<uint32_t>(pw) * 128 * (bf ? 2 : 4);
      int st = 0, uses = 0;  // stage of tile gt, earlier uses of that stage
      for (int il = 0; il < nitems && ok; ++il, w.next()) {
        if (!w.on()) continue;
        for (int j = 0; j < nt && ok; ++j, ++gt) {
          if (gt >= nst) ok = mbar_wait(bar(K_EMPTY + st), (uses - 1) & 1, abort_flag, 39);
          if (!ok) break;
          mbar_expect_tx(bar(K_FULL + st), tile_bytes);
          for (int bx = 0; bx < (pw + fpb - 1) / fpb; ++bx)
            tma_load_3d(base + sp::phi_box(st, bx, bf), &maps.phik, bar(K_FULL + st),
                        w.half() * pw + fpb * bx, w.slice * HW + j * 128, w.bh());
          if (++st == nst) {
            st = 0;
            ++uses;
          }
        }
      }
    } else if (lane == 0 && !(warp == 8 && phi_given)) {  // no K or W_k with phi_k given
      const bool kside = warp == 8;
      bool ok = true;
      int wloads = 0, wkey = -1;
      const uint32_t box_bytes = static_cast<uint32_t>(pw) * 128;  // one 64-column box
      const uint32_t ring = kside ? kKOff : kVOff;
      const int full = kside ? K_FULL : V_FULL, empty = kside ? K_EMPTY : V_EMPTY;
      sp::ItemWalk w{T, halves, P.heads, pw, leave};
      w.start(it0);
      int gt = 0, st = 0, uses = 0;  // tile index, its ring stage, earlier uses of the stage
      for (int il = 0; il < nitems && ok; ++il, w.next()) {
        if (!w.on()) continue;
        if (kside && w.wkey != wkey) {
          wkey = w.wkey;
          if (wloads > 0) ok = mbar_wait(bar(W_FREE), (wloads - 1) & 1, abort_flag, 27);
          if (!ok) break;
          // Full forward: the W_k image comes from the grid launched just
          // before this one (programmatic dependent launch).
          if (!step && wloads == 0) dependency_wait();
          // Head h's image holds its D' features as pieces of pw rows, each
          // piece two boxes of pw rows x 64 columns.
          const __nv_bfloat16* src = wk_img + static_cast<long long>(w.wkey) * pw * 128;
          mbar_expect_tx(bar(W_FULL), 2 * box_bytes);
          bulk_load(base + kWOff, src, box_bytes, bar(W_FULL));
          bulk_load(base + kWOff + 16384, src + pw * 64, box_bytes, bar(W_FULL));
          ++wloads;
        }
        const int bh = w.bh();
        const CUtensorMap* map = kside ? &maps.k : &maps.v;
        int row0 = w.slice * HW;
        if (step) {
          const long long g = seen0 - rseen + w.slice;  // global slice of this slot
          if (g < seen0) {
            map = kside ? &maps.rk : &maps.rv;
            row0 = static_cast<int>(g % P.To) * HW;
          } else {
            row0 = static_cast<int>(g - seen0) * HW;
          }
        }
        for (int j = 0; j < nt && ok; ++j, ++gt) {
          const int row = row0 + j * 128;
          if (gt >= kS) ok = mbar_wait(bar(empty + st), (uses - 1) & 1, abort_flag, kside ? 28 : 29);
          if (!ok) break;
          mbar_expect_tx(bar(full + st), 32768);
          tma_load_3d(base + ring + st * 32768, map, bar(full + st), 0, row, bh);
          tma_load_3d(base + ring + st * 32768 + 16384, map, bar(full + st), 64, row, bh);
          if (++st == kS) {
            st = 0;
            ++uses;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ================================================= psi^T MMA issuer
    if (lane == 0) {
      const uint32_t id_psi = idesc(128, 128, 1, false);  // W_k piece and K tile, K-major
      bool ok = true;
      int wwaits = 0, wkey = -1;
      // The next psi^T to issue: its tile index, item walk (on active
      // items), tile in item, K stage and earlier uses of that stage.
      sp::ItemWalk wp{T, halves, P.heads, pw, leave};
      wp.start(it0);
      if (TT > 0)
        while (!wp.on()) wp.next();
      int pgt = 0, pj = 0, pst = 0, puses = 0;
      // psi^T for token tile pgt into buffer pgt & 1: waits for its K tile,
      // for phi^T V of tile pgt - 2 to have read that buffer, and for W_k.
      auto issue_psi = [&]() -> bool {
        const int b = pgt & 1;
        if (pj == 0 && wp.wkey != wkey) {
          wkey = wp.wkey;
          if (pgt > 0) mma_commit(bar(W_FREE));  // tracks every earlier MMA
          if (!mbar_wait(bar(W_FULL), wwaits & 1, abort_flag, 30)) return false;
          ++wwaits;
        }
        if (!mbar_wait(bar(K_FULL + pst), puses & 1, abort_flag, 31)) return false;
        if (pgt >= 2 && !mbar_wait(bar(PSI_FREE + b), ((pgt - 2) >> 1) & 1, abort_flag, 32))
          return false;
        tc_fence_after();
        const uint64_t wdesc = sdesc(base + kWOff, 16, 1024);
        const uint64_t kdesc = sdesc(base + kKOff + pst * 32768, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // Descriptor start addresses are in 16-byte units (no carry: < 2^14).
          const uint64_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          mma_bf16(tmem + kColPsi + b * 128, wdesc + off, kdesc + off, id_psi, kk > 0);
        }
        mma_commit(bar(PSI_FULL + b));
        mma_commit(bar(K_EMPTY + pst));
        ++pgt;
        if (++pst == kS) {
          pst = 0;
          ++puses;
        }
        if (++pj == nt && pgt < TT) {  // on to the next active item
          pj = 0;
          do wp.next();
          while (!wp.on());
        }
        return true;
      };
      if (!phi_given)
        for (int g = 0; g < TT && ok; ++g) ok = issue_psi();
    }
    __syncwarp();
  } else if (warp == 10) {
    // ================================================= phi^T V MMA issuer
    // (a second issuing thread: its MMAs read phi^T and V and accumulate P,
    // operands the psi^T issuer never touches; each commit tracks this
    // thread's own MMAs)
    if (lane == 0) {
      const uint32_t id_pv = idesc(128, 128, 1, true);  // phi^T from TMEM, V MN-major
      bool ok = true;
      int gt = 0, vst = 0, vuses = 0;
      for (int ia = 0; ia < nactive && ok; ++ia) {  // active items
        for (int j = 0; j < nt && ok; ++j, ++gt) {
          const int b = gt & 1;
          if (j == 0 && ia >= 1)  // the epilogue has drained the previous item
            ok = mbar_wait(bar(P_FREE), (ia - 1) & 1, abort_flag, 33);
          if (ok) ok = mbar_wait(bar(PHI_FULL + b), (gt >> 1) & 1, abort_flag, 34) &&
                       mbar_wait(bar(V_FULL + vst), vuses & 1, abort_flag, 35);
          if (!ok) break;
          tc_fence_after();
          const uint64_t vdesc = sdesc(base + kVOff + vst * 32768, 16384, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + kColP, tmem + kColPhi + b * 64 + kk * 8,
                        vdesc + ((kk * 2048) >> 4), id_pv, (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(PHI_FREE + b));
          mma_commit(bar(V_EMPTY + vst));
          if (j == nt - 1) mma_commit(bar(ACC_DONE));
          if (++vst == kS) {
            vst = 0;
            ++vuses;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // ================================================= convert (thread = feature)
    const int f = tid;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    auto wait_all = [&](uint32_t b, uint32_t parity, uint32_t code) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, code));
    };
    bool ok = true;
    float bias = 0.f;
    uint64_t zacc = f2_pack(0.f, 0.f);  // z over even / odd tokens
    sp::ItemWalk w{T, halves, P.heads, pw, leave};
    w.start(it0);
    int gt = 0, vst = 0, vuses = 0, wkey = -1;
    // phi_k given: the shared-memory stage of the current tile, its uses.
    constexpr int nfst = sp::phi_stages(phi_bf16);
    int fst = 0, fuses = 0;
    for (int il = 0; il < nitems && ok; ++il, w.next()) {
      if (!w.on()) continue;
      // b_k of head h is h's D' consecutive features.
      if (w.wkey != wkey) {
        wkey = w.wkey;
        bias = f < pw && !phi_given ? P.bk[wkey * pw + f] : 0.f;
      }
      const uint64_t b2 = f2_pack(bias, bias);
      // phi_k(k) given: this thread's feature column of the item's rows.
      for (int j = 0; j < nt && ok; ++j, ++gt) {
        const int b = gt & 1;
        // psi^T of the tile in TMEM buffer b, or (phi_k given) its phi_k
        // tile in shared-memory stage b.
        ok = phi_given ? wait_all(bar(K_FULL + fst), fuses & 1, 36)
                       : wait_all(bar(PSI_FULL + b), (gt >> 1) & 1, 36);
        // phi^T buffer b is free once phi^T V of tile gt - 2 has read it.
        if (ok && gt >= 2) ok = wait_all(bar(PHI_FREE + b), ((gt - 2) >> 1) & 1, 38);
        if (!ok) break;
        tc_fence_after();
        const int nvalid = min(128, HW - j * 128);
        const uint32_t cols = lane_base + kColPsi + b * 128;
        const uint32_t pcols = lane_base + kColPhi + b * 64;
        // 32 tokens at a time: phi of tokens 32c.. becomes 16 packed columns
        // at 16c of the phi^T buffer.
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ps[32], pk[16];
          if (phi_given && phi_bf16) {
            // Feature f of tokens 32c .. 32c + 31: a column of box f / 64
            // (token-major rows of 64 bf16; a warp reads half a row).
            const __nv_bfloat16* col = reinterpret_cast<const __nv_bfloat16*>(
                                           sbase + sp::phi_box(fst, f < pw ? f >> 6 : 0, true)) +
                                       (f & 63);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int t = c * 32 + i;
              ps[i] = __float_as_uint(f < pw && t < nvalid ? __bfloat162float(col[t * 64]) : 0.f);
            }
          } else if (phi_given) {
            // Feature f of tokens 32c .. 32c + 31: a column of box f / 32
            // (token-major rows of 32 floats; a warp reads whole rows).
            const float* col = reinterpret_cast<const float*>(
                                   sbase + sp::phi_box(fst, f < pw ? f >> 5 : 0, false)) + (f & 31);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int t = c * 32 + i;
              ps[i] = __float_as_uint(f < pw && t < nvalid ? col[t * 32] : 0.f);
            }
          } else {
            REHYAT_TMEM_LD32(cols + c * 32, ps);
            tmem_wait_ld();
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            uint64_t a = f2_pack(__uint_as_float(ps[2 * i]), __uint_as_float(ps[2 * i + 1]));
            if (!phi_given) {  // phi = (psi + b)^2
              a = f2_add(a, b2);
              a = f2_fma(a, a, 0ull);
            }
            float v0, v1;
            f2_unpack(a, v0, v1);
            if (nvalid < 128) {  // tokens past the slice contribute nothing
              const int t = c * 32 + 2 * i;
              v0 = t < nvalid ? v0 : 0.f;
              v1 = t + 1 < nvalid ? v1 : 0.f;
            }
            pk[i] = pack_bf16(v0, v1);
            // z sums the same bf16-rounded values that enter phi^T V.
            zacc = f2_add(zacc, f2_pack(__uint_as_float(pk[i] << 16),
                                        __uint_as_float(pk[i] & 0xFFFF0000u)));
          }
          REHYAT_TMEM_ST16(pcols + c * 16, pk);
        }
        if (phi_given) {  // the stage's reads are done
          mbar_arrive(bar(K_EMPTY + fst));
          if (++fst == nfst) {
            fst = 0;
            ++fuses;
          }
        }
        tmem_wait_st();
        if (nvalid < 128) {
          // V rows past the slice are zeroed so that 0 * V stays 0 for any V.
          ok = wait_all(bar(V_FULL + vst), vuses & 1, 37);
          if (!ok) break;
          const int nchunks = (128 - nvalid) * 16;
          for (int i = f; i < nchunks; i += 128) {
            const int row = nvalid + (i >> 4), ch = i & 15;
            st_shared_v4(base + kVOff + vst * 32768 + (ch >> 3) * 16384 + row * 128 + (ch & 7) * 16,
                         0, 0, 0, 0);
          }
          fence_proxy_async();
        }
        tc_fence_before();
        if (!phi_given) mbar_arrive(bar(PSI_FREE + b));
        mbar_arrive(bar(PHI_FULL + b));
        if (++vst == kS) {
          vst = 0;
          ++vuses;
        }
      }
      if (ok) {
        float z0, z1;
        f2_unpack(zacc, z0, z1);
        if (f < pw) P.z[w.out_index(P.nslots) * Dp + w.half() * pw + f] = z0 + z1;
        zacc = f2_pack(0.f, 0.f);
      }
    }
  } else if (warp < 8) {
    // ================================================= epilogue (thread = feature)
    const int f = tid - 128;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    bool ok = true;
    sp::ItemWalk w{T, halves, P.heads, pw, leave};
    w.start(it0);
    int ia = 0;  // active items so far
    for (int il = 0; il < nitems && ok; ++il, w.next()) {
      if (!w.on()) continue;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(ACC_DONE), ia & 1, abort_flag, 39));
      ++ia;
      if (!ok) break;
      tc_fence_after();
      // Feature fg of the slice; the state is stored in the S^L image layout
      // (a warp writes one 128-byte row per column).
      const int fg = w.half() * pw + f;
      float* prow = P.P + w.out_index(P.nslots) * Dp * 128 + sl_feature_base(fg, 128, Dp);
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        REHYAT_TMEM_LD32(lane_base + kColP + c * 32, v);
        tmem_wait_ld();
        if (f < pw) {
#pragma unroll
          for (int i = 0; i < 32; ++i) prow[sl_column_offset(fg, c * 32 + i)] = __uint_as_float(v[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(P_FREE));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
  dependency_wait();
}

// ------------------------------------------------------------ host side
// Per-device one-time launch setup: SM count, and the dynamic shared-memory
// limit of each tensor-core kernel (the attribute is per context, so it is
// set once per device and kernel, not on every call).
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<unsigned> g_smem_set[kMaxDevices];

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <typename Kernel>
cudaError_t ensure_smem(Kernel* fn, unsigned bit, uint32_t bytes) {
  int dev = 0;
  const bool cached = cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices;
  if (cached && (g_smem_set[dev].load(std::memory_order_acquire) & (1u << bit))) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(bytes));
  if (e == cudaSuccess && cached) g_smem_set[dev].fetch_or(1u << bit, std::memory_order_release);
  return e;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3D 8-bit map over [planes][rows][128] with a 128 x 128 x 1 box (one 128-byte
// row per token), 128B swizzle.
// A given feature map [planes][rows][cols], fp32 or bf16, with boxes of 128
// bytes of columns (32 fp32 or 64 bf16) x 128 rows, unswizzled (a box lands
// as 128 rows of 128 bytes).
bool make_map_phi(CUtensorMap* m, const void* ptr, long long rows, int planes, int cols,
                  bool bf16) {
  auto fn = encode_fn();
  const int eb = bf16 ? 2 : 4;
  if (!fn || rows <= 0 || (cols * eb) % 128 != 0) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * eb,
                           static_cast<cuuint64_t>(rows) * cols * eb};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / eb), 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
            const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map8(CUtensorMap* m, const void* ptr, long long rows, int planes) {
  auto fn = encode_fn();
  if (!fn || rows <= 0) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD),
                           static_cast<cuuint64_t>(rows) * kD};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map over [planes][rows][128] with a 64 x 128 x 1 box, 128B swizzle.
bool make_map(CUtensorMap* m, const void* ptr, long long rows, int planes) {
  auto fn = encode_fn();
  if (!fn || rows <= 0) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * 2,
                           static_cast<cuuint64_t>(rows) * kD * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_state_eligible(int in_bf16, int D, int Dp) {
  return in_bf16 && D == kD && (Dp == 64 || Dp == 128 || Dp == 256) && encode_fn() != nullptr;
}

cudaError_t launch_state_tc(const PartialParams& p, const void* wk_img, cudaStream_t s) {
  StMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_map(&maps.k, p.k, p.rows_per_bh, p.BH) || !make_map(&maps.v, p.v, p.rows_per_bh, p.BH))
    return cudaErrorInvalidValue;
  if (p.seen && p.ring_rows_per_bh > 0) {
    if (!make_map(&maps.rk, p.rk, p.ring_rows_per_bh, p.BH) ||
        !make_map(&maps.rv, p.rv, p.ring_rows_per_bh, p.BH))
      return cudaErrorInvalidValue;
  } else {
    maps.rk = maps.k;
    maps.rv = maps.v;
  }
  // Persistent CTAs, each with the same number of items.
  const int sms = sm_count();
  const int per_bh = (p.seen ? p.nq_slices : p.nslots) * (p.Dp > 128 ? p.Dp / 128 : 1);
  const int total = p.BH * per_bh;
  const int per_cta = (total + sms - 1) / sms;
  const int ctas = (total + per_cta - 1) / per_cta;
  const __nv_bfloat16* wk = static_cast<const __nv_bfloat16*>(wk_img);
  if (p.phi_k != nullptr) {  // full forward with phi_k(k) given
    if (!make_map_phi(&maps.phik, p.phi_k, p.rows_per_bh, p.BH, p.Dp, p.phi_bf16 != 0))
      return cudaErrorInvalidValue;
    if (p.phi_bf16) {
      const cudaError_t e = ensure_smem(tc_state_persistent_kernel<true, true>, 10, sp::kSmemBytes);
      if (e != cudaSuccess) return e;
      tc_state_persistent_kernel<true, true><<<ctas, sp::kThreads, sp::kSmemBytes, s>>>(
          maps, p, wk, per_cta);
    } else {
      const cudaError_t e = ensure_smem(tc_state_persistent_kernel<true>, 3, sp::kSmemBytes);
      if (e != cudaSuccess) return e;
      tc_state_persistent_kernel<true><<<ctas, sp::kThreads, sp::kSmemBytes, s>>>(maps, p, wk,
                                                                                  per_cta);
    }
    return cudaGetLastError();
  }
  const cudaError_t e = ensure_smem(tc_state_persistent_kernel<false>, 0, sp::kSmemBytes);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch in both modes.  Full forward: the grid
  // before this one writes the W_k image; the K/V loads start at once and
  // the W_k load waits for that grid on the device.  Streaming fold: it reads
  // only k, v, the ring and W_k and writes only the per-slot states, so it
  // may run beside the attention kernel launched just before it.  Either way
  // the kernel waits for the earlier grid before it exits.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(sp::kThreads);
  cfg.dynamicSmemBytes = sp::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_state_persistent_kernel<false>, maps, p, wk, per_cta);
}

bool tc_attn_eligible(int in_bf16, int D, int Dp) {
  return in_bf16 && D == kD && (Dp == 64 || Dp == 128 || Dp == 256);
}

bool tc_attn_supported(const AttnParams& p) {
  if (!p.in_bf16 || p.D != kD) return false;
  if (!p.full_softmax) {
    if (!tc_attn_eligible(p.in_bf16, p.D, p.Dp)) return false;
    // phi_q given: the two-query-tile kernel reads it in its tail.
    if (p.phi_q != nullptr) {
      if (p.one_tile) return false;
    } else if (p.wq_img == nullptr) {
      return false;
    }
  }
  return encode_fn() != nullptr;
}

namespace {
struct StepSplitKey {
  int BH, HW, nq, To, sms;
  bool operator<(const StepSplitKey& o) const {
    return std::tie(BH, HW, nq, To, sms) < std::tie(o.BH, o.HW, o.nq, o.To, o.sms);
  }
};
std::mutex g_split_mu;
std::map<StepSplitKey, StepSplit> g_split_cache;

StepSplit choose_step_split(int BH, int HW, int nq_slices, int To, int sms) {
  // Pieces run as CTAs, one per SM, in work-list order; a greedy list
  // schedule of their estimated lengths on `sms` SMs gives the makespan.
  // Units: one key step of a two-tile CTA (about 2.3 us on the 30x52
  // layer).  A tile-A-only pair's step costs about 0.8 of that; a CTA's
  // prologue 1.5 steps, its tail 4.5, a split piece's tail 6.5 on average
  // (its partials, and for the last piece the merge).
  StepSplit none{1, 0};
  const int qrows = nq_slices * HW;
  const int npairs = (qrows + 2 * kBM - 1) / (2 * kBM);
  if (BH <= 0 || npairs <= 0 || sms <= 0) return none;
  const bool light = qrows - (npairs - 1) * 2 * kBM <= kBM;
  const int nfull = npairs - (light ? 1 : 0);
  const int nl = light ? BH : 0;
  const int full = BH * nfull;
  const int ntb = (qrows + kBN - 1) / kBN;
  const int nt = (To * HW + kBN - 1) / kBN + ntb;
  if (full == 0 || nl + full > 3 * sms) return none;
  std::vector<double> load(static_cast<size_t>(sms));
  auto makespan = [&](int ks, int whole) {
    std::priority_queue<double, std::vector<double>, std::greater<double>> q;
    for (int i = 0; i < sms; ++i) q.push(0.0);
    auto put = [&](double cost) {
      const double t0 = q.top();
      q.pop();
      q.push(t0 + cost);
    };
    for (int i = 0; i < nl; ++i) put(1.5 + 0.8 * nt + 4.5);
    for (int i = 0; i < whole; ++i) put(1.5 + nt + 4.5);
    for (int i = whole; i < full; ++i)
      for (int pc = 0; pc < ks; ++pc)
        put(1.5 + static_cast<double>((pc + 1) * nt / ks - pc * nt / ks) + 6.5);
    double mx = 0.0;
    while (!q.empty()) {
      mx = q.top() > mx ? q.top() : mx;
      q.pop();
    }
    return mx;
  };
  const double base = makespan(1, full);
  StepSplit best = none;
  double best_t = base;
  const int cand[] = {0, sms - nl, sms, 2 * sms - nl, 2 * sms};
  for (int ks = 2; ks <= 4 && ks <= ntb; ++ks)
    for (int w : cand) {
      if (w < 0 || w >= full) continue;
      const double tk = makespan(ks, w);
      if (tk < best_t) {
        best_t = tk;
        best = StepSplit{ks, w};
      }
    }
  return best_t < 0.97 * base ? best : none;
}
}  // namespace

StepSplit attn_step_split(int BH, int HW, int nq_slices, int To, int sms) {
  const StepSplitKey key{BH, HW, nq_slices, To, sms};
  std::lock_guard<std::mutex> lock(g_split_mu);
  auto it = g_split_cache.find(key);
  if (it != g_split_cache.end()) return it->second;
  const StepSplit r = choose_step_split(BH, HW, nq_slices, To, sms);
  if (g_split_cache.size() < 4096) g_split_cache.emplace(key, r);
  return r;
}

size_t attn_split_part_bytes(int BH, int HW, int nq_slices, StepSplit sp) {
  if (sp.ksplit <= 1) return 0;
  const int qrows = nq_slices * HW;
  const int npairs = (qrows + 2 * kBM - 1) / (2 * kBM);
  const bool light = qrows - (npairs - 1) * 2 * kBM <= kBM;
  const long long full = static_cast<long long>(BH) * (npairs - (light ? 1 : 0));
  if (sp.whole < 0 || sp.whole >= full) return 0;
  return static_cast<size_t>(full - sp.whole) * sp.ksplit * 2 * a2::kPartVec * kBM * 16;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s) {
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_map(&maps.q, p.q, p.rows_per_bh, p.BH) || !make_map(&maps.k, p.k, p.rows_per_bh, p.BH) ||
      !make_map(&maps.v, p.v, p.rows_per_bh, p.BH))
    return cudaErrorInvalidValue;
  if (p.seen) {
    // Ring of T_o slices; with T_o = 0 the ring is never read (any valid map).
    const long long ring_rows = p.ring_rows_per_bh > 0 ? p.ring_rows_per_bh : 0;
    if (ring_rows > 0) {
      if (!make_map(&maps.rk, p.rk, ring_rows, p.BH) || !make_map(&maps.rv, p.rv, ring_rows, p.BH))
        return cudaErrorInvalidValue;
    } else {
      maps.rk = maps.k;
      maps.rv = maps.v;
    }
  }
  const int qrows_max = p.seen ? p.nq_slices * p.HW : (p.Tc < p.T ? p.Tc : p.T) * p.HW;
  const bool two_tiles = !p.one_tile;
  cudaError_t e;
  if (p.q8 != nullptr) {  // fp8 softmax variant (full forward, two-tile kernel only)
    if (!two_tiles || p.seen || !make_map8(&maps.q8, p.q8, p.rows_per_bh, p.BH) ||
        !make_map8(&maps.k8, p.k8, p.rows_per_bh, p.BH))
      return cudaErrorInvalidValue;
    e = ensure_smem(tc_attn2_kernel<true>, 5, a2::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid((qrows_max + 2 * kBM - 1) / (2 * kBM), p.nchunks, p.BH);
    tc_attn2_kernel<true><<<grid, a2::kThreads, a2::kSmemBytes, s>>>(
        maps, p, static_cast<const __nv_bfloat16*>(p.wq_img));
  } else if (two_tiles) {
    e = ensure_smem(tc_attn2_kernel<false>, 1, a2::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid((qrows_max + 2 * kBM - 1) / (2 * kBM), p.nchunks, p.BH);
    if (p.seen && p.ksplit > 1) {
      // Work list: the tile-A-only pairs, kwhole whole two-tile pairs, then
      // ksplit pieces for each remaining two-tile pair.
      const int npairs = static_cast<int>(grid.x);
      const bool light = qrows_max - (npairs - 1) * 2 * kBM <= kBM;
      const int full = p.BH * (npairs - (light ? 1 : 0));
      if (!p.part || !p.part_cnt || p.nchunks != 1 || p.kwhole < 0 || p.kwhole >= full)
        return cudaErrorInvalidValue;
      grid = dim3((light ? p.BH : 0) + p.kwhole + (full - p.kwhole) * p.ksplit, 1, 1);
    }
    tc_attn2_kernel<false><<<grid, a2::kThreads, a2::kSmemBytes, s>>>(
        maps, p, static_cast<const __nv_bfloat16*>(p.wq_img));
  } else {
    e = ensure_smem(tc_attn_kernel, 2, kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid((qrows_max + kBM - 1) / kBM, p.nchunks, p.BH);
    tc_attn_kernel<<<grid, kThreads, kSmemBytes, s>>>(
        maps, p, static_cast<const __nv_bfloat16*>(p.wq_img));
  }
  return cudaGetLastError();
}

}  // namespace rehyat

// The general feature map's and the backward's tensor-core kernels share
// this unit's helpers.
#include "tc_phi_mlp.cuh"
#include "tc_attn_bwd.cuh"

namespace rehyat {
cudaError_t read_den_rows_simt(unsigned long long* rows, int reset);
}

extern "C" rehyat_status rehyat_denominator_report(unsigned long long* rows, int reset) {
  if (!rows) return REHYAT_ERR_INVALID_ARG;
  unsigned long long tc = 0, simt = 0;
  if (cudaMemcpyFromSymbol(&tc, rehyat::rehyat_tc_den_rows, sizeof(tc)) != cudaSuccess ||
      rehyat::read_den_rows_simt(&simt, reset) != cudaSuccess)
    return REHYAT_ERR_CUDA;
  if (reset) {
    const unsigned long long zero = 0;
    if (cudaMemcpyToSymbol(rehyat::rehyat_tc_den_rows, &zero, sizeof(zero)) != cudaSuccess)
      return REHYAT_ERR_CUDA;
  }
  *rows = tc + simt;
  return REHYAT_OK;
}

extern "C" rehyat_status rehyat_device_error_flags(unsigned* flags, int reset) {
  if (!flags) return REHYAT_ERR_INVALID_ARG;
  if (cudaMemcpyFromSymbol(flags, rehyat::rehyat_tc_error, sizeof(unsigned)) != cudaSuccess)
    return REHYAT_ERR_CUDA;
  if (reset) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(rehyat::rehyat_tc_error, &zero, sizeof(unsigned)) != cudaSuccess)
      return REHYAT_ERR_CUDA;
  }
  return REHYAT_OK;
}
