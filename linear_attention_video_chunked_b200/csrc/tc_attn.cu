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
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "internal.h"
#include "layout.cuh"

namespace rehyat {

__device__ unsigned int rehyat_tc_error = 0;

namespace {

constexpr int kD = 128;          // head width handled here
constexpr int kBM = 128;         // query rows per CTA
constexpr int kBN = 128;         // keys per tile
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;

// Shared memory map (offsets from a 1024-aligned base).
constexpr uint32_t kQOff = 0;                        // Q: 2 boxes x 16 KB
constexpr uint32_t kStageOff = 32768;                // 2 stages x (K 32 KB + V 32 KB)
constexpr uint32_t kStageBytes = 65536;
constexpr uint32_t kPOff = kStageOff + 2 * kStageBytes;  // P: 2 boxes x 16 KB
constexpr uint32_t kBarOff = kPOff + 32768;
// Tail reuse of the stage/P region.
constexpr uint32_t kWOff = kStageOff;                // phi_q weight piece (<= 32 KB)
constexpr uint32_t kSLOff = kStageOff + 32768;       // S^L piece (<= 64 KB)
constexpr uint32_t kPhiOff = kStageOff + 98304;      // phi_q(q) piece fp32 (<= 64 KB)
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;  // + alignment slack

// Barrier slots (8 bytes each).
enum {
  B_Q_FULL = 0, B_K_FULL = 1, B_V_FULL = 3, B_KV_EMPTY = 5, B_S_FULL = 7, B_S_FREE = 9,
  B_P_FULL = 11, B_PV_DONE = 12, B_TAIL_FULL = 13, B_PHI_DONE = 14, B_PHI_READY = 15,
  B_READ_DONE = 16, B_COUNT = 17
};
constexpr uint32_t kTmemSlot = kBarOff + 8 * B_COUNT;       // u32: TMEM base address
constexpr uint32_t kAbortSlot = kTmemSlot + 4;              // u32: abort flag

constexpr uint32_t kColS0 = 0, kColO = 256, kColAL = 384;

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at the boost clock

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on the phase with the given parity.  On timeout: record the
// barrier in the global error word, raise the CTA abort flag, return false.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                                       uint32_t code) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 255u) == 255u) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        atomicOr(&rehyat_tc_error, 1u << (code & 31));
        *abort_flag = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// UMMA shared-memory descriptor: 128-byte swizzle, version 1 (sm_100).
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr & 0x3FFFFu) >> 4) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: fp32 accumulate, A K-major, A/B format fmt
// (1 = bf16, 2 = tf32), B K-major or MN-major.
__host__ __device__ constexpr uint32_t idesc(int M, int N, uint32_t fmt, bool b_mn_major) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(accumulate));
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

#define REHYAT_TMEM_LD32(taddr, r)                                                              \
  asm volatile(                                                                                \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "  \
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "  \
      "%28, %29, %30, %31}, [%32];"                                                            \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),    \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),             \
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),          \
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),          \
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),          \
        "=r"(r[31])                                                                            \
      : "r"(taddr))

#define REHYAT_TMEM_ST32(taddr, r)                                                              \
  asm volatile(                                                                                \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, " \
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "  \
      "%28, %29, %30, %31, %32};" ::"r"(taddr),                                                \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),  \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),        \
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),      \
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),      \
      "r"(r[29]), "r"(r[30]), "r"(r[31]))

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// --------------------------------------------------------------- kernel
struct TcMaps {
  CUtensorMap q, k, v, rk, rv;
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
    const uint32_t counts[B_COUNT] = {1, 1, 1, 1, 1, 1, 1, 1, 1, kSoftmaxThreads,
                                      kSoftmaxThreads, kSoftmaxThreads, 1, 1, 1,
                                      kSoftmaxThreads, 1};
    for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), counts[i]);
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
        const int s = j & 1;
        if (j >= 2) ok = mbar_wait(bar(B_KV_EMPTY + s), ((j - 2) >> 1) & 1, abort_flag, 1);
        if (!ok) break;
        const TileSrc src = tile_src(j);
        const uint32_t kdst = base + kStageOff + s * kStageBytes;
        const uint32_t vdst = kdst + 32768;
        mbar_expect_tx(bar(B_K_FULL + s), 32768);
        tma_load_3d(kdst, src.map_k, bar(B_K_FULL + s), 0, src.row, bh);
        tma_load_3d(kdst + 16384, src.map_k, bar(B_K_FULL + s), 64, src.row, bh);
        mbar_expect_tx(bar(B_V_FULL + s), 32768);
        tma_load_3d(vdst, src.map_v, bar(B_V_FULL + s), 0, src.row, bh);
        tma_load_3d(vdst + 16384, src.map_v, bar(B_V_FULL + s), 64, src.row, bh);
      }
      // Readout operands, one feature piece at a time, into the freed stages.
      const uint32_t wbytes = static_cast<uint32_t>(pw) * kD * 2;
      const uint32_t slbytes = static_cast<uint32_t>(pw) * kD * 4;
      for (int pc = 0; pc < npieces && ok; ++pc) {
        if (pc == 0)
          ok = mbar_wait(bar(B_PV_DONE), (nt - 1) & 1, abort_flag, 2);
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
        if (!mbar_wait(bar(B_K_FULL + s), (i >> 1) & 1, abort_flag, 5)) return false;
        if (i >= 2 && !mbar_wait(bar(B_S_FREE + s), ((i - 2) >> 1) & 1, abort_flag, 6))
          return false;
        tc_fence_after();
        const uint32_t kaddr = base + kStageOff + s * kStageBytes;
        const uint32_t d = tmem + kColS0 + s * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16(d, sdesc(base + kQOff + off, 16, 1024), sdesc(kaddr + off, 16, 1024), id_qk,
                   kk > 0);
        }
        mma_commit(bar(B_S_FULL + s));
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
        const uint32_t vaddr = base + kStageOff + s * kStageBytes + 32768;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = sdesc(base + kPOff + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc(vaddr + kk * 2048, 16384, 1024);
          mma_bf16(tmem + kColO, a, b, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(B_PV_DONE));
        mma_commit(bar(B_KV_EMPTY + s));
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
    for (int j = 0; j < nt && ok; ++j) {
      const int s = j & 1;
      ok = mbar_wait(bar(B_S_FULL + s), (j >> 1) & 1, abort_flag, 11);
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
      float x[128];
      tc_fence_before();
      mbar_arrive(bar(B_S_FREE + s));
      const int nvalid = tile_src(j).nvalid;
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        x[i] = (i < nvalid) ? __uint_as_float(xr[i]) * P.scale_log2 : -INFINITY;
        mt = fmaxf(mt, x[i]);
      }
      m_max = fmaxf(m_max, mt);
      float alpha = 1.f;
      const bool rescale = m_max > m_used + 8.f;
      if (rescale) {
        alpha = ex2(m_used - m_max);  // 0 on the first tile
        m_used = m_max;
      }
      uint32_t pk[64];
      float lsum = 0.f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float p0 = ex2(x[2 * i] - m_used);
        const float p1 = ex2(x[2 * i + 1] - m_used);
        pk[i] = pack_bf16(p0, p1);
        lsum += __uint_as_float(pk[i] << 16) + __uint_as_float(pk[i] & 0xFFFF0000u);
      }
      l = l * alpha + lsum;
      if (j > 0) {
        ok = mbar_wait(bar(B_PV_DONE), (j - 1) & 1, abort_flag, 12);
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
        ok = mbar_wait(bar(B_V_FULL + s), (j >> 1) & 1, abort_flag, 13);
        if (!ok) break;
        if (r >= nvalid) {
          const uint32_t vrow = base + kStageOff + s * kStageBytes + 32768 + r * 128;
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
      ok = mbar_wait(bar(B_PHI_DONE), pc & 1, abort_flag, 14);
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
        ok = mbar_wait(bar(B_READ_DONE), (npieces - 1) & 1, abort_flag, 15);
      else
        ok = mbar_wait(bar(B_PV_DONE), (nt - 1) & 1, abort_flag, 15);
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

// ------------------------------------------------------------ host side
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

bool tc_attn_eligible(int in_bf16, int D, int Dp) {
  return in_bf16 && D == kD && (Dp == 64 || Dp == 128 || Dp == 256);
}

bool tc_attn_supported(const AttnParams& p) {
  if (!p.in_bf16 || p.D != kD) return false;
  if (!p.full_softmax && (!tc_attn_eligible(p.in_bf16, p.D, p.Dp) || p.wq_img == nullptr))
    return false;
  return encode_fn() != nullptr;
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
  cudaError_t e = cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int qrows_max = p.seen ? p.nq_slices * p.HW : (p.Tc < p.T ? p.Tc : p.T) * p.HW;
  dim3 grid((qrows_max + kBM - 1) / kBM, p.nchunks, p.BH);
  tc_attn_kernel<<<grid, kThreads, kSmemBytes, s>>>(
      maps, p, static_cast<const __nv_bfloat16*>(p.wq_img));
  return cudaGetLastError();
}

}  // namespace rehyat
