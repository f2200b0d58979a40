// Tensor-core general feature map of ReHyAt for B200 (sm_100a).
//
// Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
// Transformers" (papernotes.org note), Method, Key design 3: phi maps a head's
// query or key through a light per-head embedding network whose output psi
// is cut into P equal parts, part i raised to the power i:
//   psi = GELU(x W_a + b_a) W_b + b_b,  GELU(u) = u * Phi(u) (exact form),
//   phi = [psi_1^1, ..., psi_P^P].
//
// One persistent CTA per SM walks 128-token tiles of (head, batch, tile)
// order, so a CTA changes weights at most a few times.  Per tile, the hidden
// layer is computed in pieces of 128 columns:
//   H_j   = X W_a[:, j]          tcgen05 (bf16 operands, fp32 in TMEM)
//   G_j   = GELU(H_j + b_a)      converter warps, rounded to bf16 in place
//   Psi  += G_j W_b[j, :]         tcgen05 with G_j read from TMEM (A operand)
// then the epilogue warps add b_b, raise each part to its power and store
// phi in fp32.  H has two TMEM buffers, so the product of piece j + 1 runs
// while piece j is converted; Psi has two, so one tile is stored while the
// next accumulates.
//
// Roles (448 threads):
//   warps 0-7   converters: warp w reads TMEM lanes 32 (w mod 4) .. (the
//               tile's rows) and hidden columns 64 (w / 4) .. of a piece;
//   warps 8-11  epilogue: thread = token row, all D' columns;
//   warp 12     TMA producer (one lane): X tiles, weight images;
//   warp 13     MMA issuer (one lane) and TMEM owner.
// TMEM (512 columns): H [0,128) [128,256), Psi [256,384) [384,512).
// Shared memory: X tile (32 KB), then the bf16 images of W_a^T and W_b^T of
// the current head (layout.cuh, kpiece_img_index), then the barriers.
//
// This file is part of the translation unit of tc_kernels.cu (it shares the
// wait helpers, the error word and the tensor-map helpers defined there).

namespace rehyat {
namespace {

namespace mlp {
constexpr int kThreads = 448;
constexpr int kEpiWarp0 = 8, kProducerWarp = 12, kMmaWarp = 13;
constexpr uint32_t kXOff = 0, kWOff = 32768;
enum { X_FULL = 0, X_EMPTY = 1, W_FULL = 2, W_FREE = 3, H_FULL = 4, PACKED = 6, PSI_FULL = 8,
       PSI_FREE = 10, NBAR = 12 };
constexpr uint32_t kColH = 0, kColPsi = 256;
constexpr uint32_t kMaxSmem = 232448;  // opt-in dynamic shared memory per block

// Bytes of one head's weight images: W_a^T [D_h][128] and W_b^T [D'][D_h].
__host__ __device__ constexpr uint32_t w_bytes(int Dh, int Dp) {
  return static_cast<uint32_t>(Dh) * 256u + static_cast<uint32_t>(Dp) * Dh * 2u;
}
__host__ __device__ constexpr uint32_t bar_off(int Dh, int Dp) { return kWOff + w_bytes(Dh, Dp); }
__host__ __device__ constexpr uint32_t smem_bytes(int Dh, int Dp) {
  return bar_off(Dh, Dp) + 256u + 1024u;  // barriers, TMEM slot, abort flag; alignment slack
}

struct Args {
  const __nv_bfloat16* img;  // [heads][w_bytes / 2] weight images
  const float* ba;           // [heads][Dh]
  const float* bb;           // [heads][Dp]
  void* phi;                 // [B*heads][N][Dp], fp32 or (phi_bf16) bf16
  long long N;
  int batch, heads, Dh, Dp, parts, ntile, tiles_per_cta, phi_bf16;
};

// Tile it of the walk: it = (h * batch + b) * ntile + tile.
struct Tile {
  int h, b, tile;
};
__device__ __forceinline__ Tile tile_of(int it, int batch, int ntile) {
  Tile t;
  const int hb = it / ntile;
  t.tile = it - hb * ntile;
  t.h = hb / batch;
  t.b = hb - t.h * batch;
  return t;
}

// GELU(u) = u Phi(u) with Phi(u) = (1 + erf(u / sqrt 2)) / 2 and erf from
// Abramowitz & Stegun, Handbook of Mathematical Functions, 7.1.28: for
// x >= 0, erf(x) = 1 - 1 / (1 + a1 x + a2 x^2 + ... + a6 x^6)^16 with
// |error| <= 3e-7 -- far below the bf16 rounding the result gets next.
// With r = 1 / poly^16, Phi(u) = 1 - r/2 for u >= 0 and r/2 for u < 0 (no
// cancellation in the tail; poly^16 overflows to +inf far out, where r = 0).
constexpr float kErfA1 = 0.0705230784f, kErfA2 = 0.0422820123f, kErfA3 = 0.0092705272f;
constexpr float kErfA4 = 0.0001520143f, kErfA5 = 0.0002765672f, kErfA6 = 0.0000430638f;

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// GELU of two values at once on packed fp32 pairs (sm_100 f32x2 FMA / MUL),
// rounded to a bf16 pair, written as
//   GELU(u) = max(u, 0) - |u| r / 2,  r = 1 / poly(|u| / sqrt 2)^16,
// which is u (1 - r/2) for u >= 0 and u r / 2 for u < 0.  One MUFU
// reciprocal per value, about ten FMA-pipe instructions per pair.
__device__ __forceinline__ uint32_t gelu2_bf16(float u0, float u1) {
  const uint64_t u = f2_pack(u0, u1);
  const uint64_t au = u & 0x7FFFFFFF7FFFFFFFull;  // |u| of both
  const uint64_t x = f2_mul(au, f2_pack(0.70710678118654752f, 0.70710678118654752f));
  auto c2 = [](float c) { return f2_pack(c, c); };
  uint64_t poly = f2_fma(c2(kErfA6), x, c2(kErfA5));
  poly = f2_fma(poly, x, c2(kErfA4));
  poly = f2_fma(poly, x, c2(kErfA3));
  poly = f2_fma(poly, x, c2(kErfA2));
  poly = f2_fma(poly, x, c2(kErfA1));
  poly = f2_fma(poly, x, c2(1.f));
  poly = f2_mul(poly, poly);  // ^2
  poly = f2_mul(poly, poly);  // ^4
  poly = f2_mul(poly, poly);  // ^8
  poly = f2_mul(poly, poly);  // ^16
  float p0, p1, r0, r1;
  f2_unpack(poly, p0, p1);
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(p0));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r1) : "f"(p1));
  const uint64_t t = f2_mul(au, f2_pack(r0, r1));
  const uint64_t g = f2_fma(t, c2(-0.5f), f2_pack(fmaxf(u0, 0.f), fmaxf(u1, 0.f)));
  float g0, g1;
  f2_unpack(g, g0, g1);
  return pack_bf16(g0, g1);
}

// tcgen05.ld of 16 lanes x 256 bits, four times along the columns (32
// columns): thread t holds, for repetition r, rows t/4 and t/4 + 8 of the 16
// lanes at columns 8 r + 2 (t mod 4) and + 1 -- four consecutive threads hold
// 8 consecutive columns of a row, so their stores fill whole 32-byte sectors.
#define REHYAT_TMEM_LD16x256_X4(taddr, r)                                                       \
  asm volatile(                                                                                \
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "  \
      "%11, %12, %13, %14, %15}, [%16];"                                                       \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),    \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),             \
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])                                                  \
      : "r"(taddr))

// Epilogue of one warp's 32 tile rows (TMEM lane quadrant at tq): psi = Psi +
// b_b over the D' columns, part i (columns i W .. (i + 1) W - 1, W = D' / P)
// raised to the power i + 1, stored as fp32 rows of out (row 0 = the warp's
// first row, `rows` of them valid).  kDp, kP > 0: the part width is a
// compile-time constant and the power is applied with kP - 1 predicated
// products; kP = 0: any P (a division per value).
// out: fp32 [rows][Dp], or bf16 (round to nearest even) when kBf16.
template <int kDp, int kP, bool kBf16>
__device__ __forceinline__ void store_rows(void* out, const float* bias, uint32_t tq, int rows,
                                           int Dp, int parts) {
  const int dp = kDp > 0 ? kDp : Dp;
  const int width = kP > 0 ? dp / kP : Dp / parts;
  const int t = threadIdx.x & 31;
#pragma unroll 1
  for (int lh = 0; lh < 2; ++lh) {
    const int ra = 16 * lh + (t >> 2), rb = ra + 8;
#pragma unroll 1
    for (int c0 = 0; c0 < dp; c0 += 32) {
      uint32_t r[16];
      REHYAT_TMEM_LD16x256_X4(tq + (static_cast<uint32_t>(16 * lh) << 16) + c0, r);
      asm volatile("tcgen05.wait::ld.sync.aligned;"
                   : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                     "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                     "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                   :
                   : "memory");
#pragma unroll
      for (int rep = 0; rep < 4; ++rep) {
        const int c = c0 + 8 * rep + 2 * (t & 3);
        const float2 b2 = __ldg(reinterpret_cast<const float2*>(bias + c));
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = __uint_as_float(r[4 * rep + e]) + ((e & 1) ? b2.y : b2.x);
          const int pw = (c + (e & 1)) / width + 1;
          float y = x;
          if (kP > 0) {
#pragma unroll
            for (int m = 1; m < kP; ++m)
              if (m < pw) y *= x;
          } else {
            for (int m = 1; m < pw; ++m) y *= x;
          }
          v[e] = y;
        }
        if (kBf16) {
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
          if (ra < rows)
            *reinterpret_cast<uint32_t*>(o + static_cast<long long>(ra) * dp + c) = pack_bf16(v[0], v[1]);
          if (rb < rows)
            *reinterpret_cast<uint32_t*>(o + static_cast<long long>(rb) * dp + c) = pack_bf16(v[2], v[3]);
        } else {
          float* o = static_cast<float*>(out);
          if (ra < rows)
            *reinterpret_cast<float2*>(o + static_cast<long long>(ra) * dp + c) = make_float2(v[0], v[1]);
          if (rb < rows)
            *reinterpret_cast<float2*>(o + static_cast<long long>(rb) * dp + c) = make_float2(v[2], v[3]);
        }
      }
    }
  }
}
}  // namespace mlp

__global__ void __launch_bounds__(mlp::kThreads, 1)
    tc_phi_mlp_kernel(const __grid_constant__ CUtensorMap xmap, const mlp::Args a) {
  // Local names shadow the attention kernel's constants of the same names.
  constexpr int kProducerWarp = mlp::kProducerWarp, kMmaWarp = mlp::kMmaWarp;
  constexpr int kEpiWarp0 = mlp::kEpiWarp0;
  constexpr uint32_t kXOff = mlp::kXOff, kWOff = mlp::kWOff;
  constexpr uint32_t kColH = mlp::kColH, kColPsi = mlp::kColPsi;
  using mlp::X_FULL;
  using mlp::X_EMPTY;
  using mlp::W_FULL;
  using mlp::W_FREE;
  using mlp::H_FULL;
  using mlp::PACKED;
  using mlp::PSI_FULL;
  using mlp::PSI_FREE;
  using mlp::NBAR;
  using mlp::Tile;
  using mlp::tile_of;
  using mlp::bar_off;
  using mlp::w_bytes;
  using mlp::gelu2_bf16;
  using mlp::store_rows;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const int Dh = a.Dh, Dp = a.Dp;
  const uint32_t boff = bar_off(Dh, Dp);
  auto bar = [&](int i) { return base + boff + 8u * i; };
  const uint32_t tmem_slot = boff + 8u * NBAR;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sbase + tmem_slot + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int J = Dh >> 7;  // hidden pieces of 128
  const int total = a.heads * a.batch * a.ntile;
  const int it0 = blockIdx.x * a.tiles_per_cta;
  const int it1 = min(total, it0 + a.tiles_per_cta);
  if (it0 >= it1) return;

  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) {
      uint32_t count = 1;
      if (i == PACKED || i == PACKED + 1) count = 8;      // one arrive per converter warp
      if (i == PSI_FREE || i == PSI_FREE + 1) count = 4;  // one per epilogue warp
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     base + tmem_slot),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + tmem_slot);

  if (warp == kProducerWarp) {
    // ================================================= TMA producer
    if (lane == 0) {
      bool ok = true;
      int wl = 0, head = -1;
      const uint32_t wb = w_bytes(Dh, Dp);
      for (int it = it0, tl = 0; it < it1 && ok; ++it, ++tl) {
        const Tile t = tile_of(it, a.batch, a.ntile);
        if (t.h != head) {
          head = t.h;
          if (wl > 0) ok = mbar_wait(bar(W_FREE), (wl - 1) & 1, abort_flag, 40);
          if (!ok) break;
          const uint8_t* src = reinterpret_cast<const uint8_t*>(a.img) +
                               static_cast<long long>(t.h) * wb;
          mbar_expect_tx(bar(W_FULL), wb);
          for (uint32_t o = 0; o < wb; o += 32768u)
            bulk_load(base + kWOff + o, src + o, wb - o < 32768u ? wb - o : 32768u, bar(W_FULL));
          ++wl;
        }
        if (tl > 0) ok = mbar_wait(bar(X_EMPTY), (tl - 1) & 1, abort_flag, 41);
        if (!ok) break;
        const int plane = t.b * a.heads + t.h;
        mbar_expect_tx(bar(X_FULL), 32768);
        tma_load_3d(base + kXOff, &xmap, bar(X_FULL), 0, t.tile * 128, plane);
        tma_load_3d(base + kXOff + 16384, &xmap, bar(X_FULL), 64, t.tile * 128, plane);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ================================================= MMA issuer
    if (lane == 0) {
      const uint32_t id1 = idesc(128, 128, 1, false);  // X . W_a piece, both K-major
      const uint32_t id2 = idesc(128, Dp, 1, false);   // G (TMEM) . W_b piece
      const uint64_t xdesc = sdesc(base + kXOff, 16, 1024);
      const uint32_t wb_off = kWOff + static_cast<uint32_t>(Dh) * 256u;
      bool ok = true;
      int wwaits = 0, head = -1;
      int pend = -1, pend_tl = 0, pend_j = 0;  // piece whose second product is not issued
      // Second product of piece g (tile tl, piece j): waits for its GELU
      // output, and at j = 0 for the epilogue to have drained Psi buffer
      // tl & 1 (tile tl - 2).
      auto issue_g2 = [&](int g, int tl, int j) -> bool {
        const int b = g & 1, pb = tl & 1;
        if (!mbar_wait(bar(PACKED + b), (g >> 1) & 1, abort_flag, 42)) return false;
        if (j == 0 && tl >= 2 && !mbar_wait(bar(PSI_FREE + pb), ((tl - 2) >> 1) & 1, abort_flag, 43))
          return false;
        tc_fence_after();
        const uint64_t bdesc = sdesc(base + wb_off + static_cast<uint32_t>(j * Dp) * 256u, 16, 1024);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          // k-step s: hidden 16 s .. of the piece; the converter half s / 4
          // left its 32 packed columns at the start of its 64 input columns.
          const uint32_t acol = tmem + kColH + b * 128 + (s >> 2) * 64 + (s & 3) * 8;
          const uint64_t off = static_cast<uint64_t>(((s >> 2) * Dp * 128 + (s & 3) * 32) >> 4);
          mma_bf16_ts(tmem + kColPsi + pb * 128, acol, bdesc + off, id2,
                      (j > 0 || s > 0) ? 1u : 0u);
        }
        if (j == J - 1) mma_commit(bar(PSI_FULL + pb));
        return true;
      };
      int gp = 0;
      for (int it = it0, tl = 0; it < it1 && ok; ++it, ++tl) {
        const Tile t = tile_of(it, a.batch, a.ntile);
        for (int j = 0; j < J && ok; ++j, ++gp) {
          if (j == 0) {
            if (t.h != head) {
              // Finish every product that reads the old weights, then let
              // the producer replace them.
              if (pend >= 0) {
                ok = issue_g2(pend, pend_tl, pend_j);
                pend = -1;
                if (!ok) break;
                mma_commit(bar(W_FREE));
              }
              head = t.h;
              ok = mbar_wait(bar(W_FULL), wwaits & 1, abort_flag, 44);
              ++wwaits;
              if (!ok) break;
            }
            ok = mbar_wait(bar(X_FULL), tl & 1, abort_flag, 45);
            if (!ok) break;
          }
          tc_fence_after();
          // H buffer gp & 1 was last read by the second product of piece
          // gp - 2, issued before this point (one thread's tcgen05 ops run
          // in order), after its converters had finished with it.
          const int b = gp & 1;
          const uint64_t wdesc = sdesc(base + kWOff + static_cast<uint32_t>(j) * 32768u, 16, 1024);
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint64_t off = static_cast<uint64_t>(((s >> 2) * 16384 + (s & 3) * 32) >> 4);
            mma_bf16(tmem + kColH + b * 128, xdesc + off, wdesc + off, id1, s > 0 ? 1u : 0u);
          }
          mma_commit(bar(H_FULL + b));
          if (j == J - 1) mma_commit(bar(X_EMPTY));
          if (pend >= 0) ok = issue_g2(pend, pend_tl, pend_j);
          pend = gp;
          pend_tl = tl;
          pend_j = j;
        }
      }
      if (ok && pend >= 0) issue_g2(pend, pend_tl, pend_j);
    }
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ================================================= converters
    const int hc = warp >> 2;  // column half of a piece
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    bool ok = true;
    int gp = 0;
    for (int it = it0; it < it1 && ok; ++it) {
      const Tile t = tile_of(it, a.batch, a.ntile);
      for (int j = 0; j < J; ++j, ++gp) {
        const int b = gp & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(H_FULL + b), (gp >> 1) & 1, abort_flag, 46));
        if (!ok) break;
        tc_fence_after();
        const uint32_t col = lane_base + kColH + b * 128 + hc * 64;
        // b_a of these 64 hidden columns (16-byte aligned; the same address
        // in every lane, so each load is a broadcast).
        const float4* bias4 = reinterpret_cast<const float4*>(
            a.ba + static_cast<long long>(t.h) * Dh + j * 128 + hc * 64);
        // Both 32-column chunks are loaded up front.  Columns 32c..32c+31
        // become packed columns 16c..16c+15, which this thread has already
        // read (chunk 0 writes over its own input).
        uint32_t r0[32], r1[32];
        REHYAT_TMEM_LD32(col, r0);
        REHYAT_TMEM_LD32(col + 32, r1);
        auto convert = [&](const uint32_t* r, uint32_t dst, const float4* b) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 b4 = __ldg(b + i);
            pk[2 * i] = gelu2_bf16(__uint_as_float(r[4 * i]) + b4.x,
                                   __uint_as_float(r[4 * i + 1]) + b4.y);
            pk[2 * i + 1] = gelu2_bf16(__uint_as_float(r[4 * i + 2]) + b4.z,
                                       __uint_as_float(r[4 * i + 3]) + b4.w);
          }
          REHYAT_TMEM_ST16(dst, pk);
        };
        REHYAT_TMEM_WAIT_LD32(r0);
        REHYAT_TMEM_WAIT_LD32(r1);
        convert(r0, col, bias4);
        convert(r1, col + 16, bias4 + 8);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(PACKED + b));
      }
    }
  } else {
    // ================================================= epilogue (thread = token)
    const int q = warp - kEpiWarp0;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    bool ok = true;
    int tl = 0;
    for (int it = it0; it < it1 && ok; ++it, ++tl) {
      const Tile t = tile_of(it, a.batch, a.ntile);
      const int pb = tl & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(PSI_FULL + pb), (tl >> 1) & 1, abort_flag, 47));
      if (!ok) break;
      tc_fence_after();
      const long long row0 = static_cast<long long>(t.tile) * 128 + q * 32;
      const int rows = static_cast<int>(min(32LL, a.N - row0));
      const long long o0 = (static_cast<long long>(t.b * a.heads + t.h) * a.N + row0) * Dp;
      void* out = a.phi_bf16 ? static_cast<void*>(static_cast<__nv_bfloat16*>(a.phi) + o0)
                             : static_cast<void*>(static_cast<float*>(a.phi) + o0);
      const float* bias = a.bb + static_cast<long long>(t.h) * Dp;
      const uint32_t tq = lane_base + kColPsi + pb * 128;
      const int P = a.parts;
      if (a.phi_bf16) {
        if (Dp == 128 && P == 2) store_rows<128, 2, true>(out, bias, tq, rows, Dp, P);
        else if (Dp == 128 && P == 1) store_rows<128, 1, true>(out, bias, tq, rows, Dp, P);
        else if (Dp == 64 && P == 2) store_rows<64, 2, true>(out, bias, tq, rows, Dp, P);
        else store_rows<0, 0, true>(out, bias, tq, rows, Dp, P);
      } else {
        if (Dp == 128 && P == 2) store_rows<128, 2, false>(out, bias, tq, rows, Dp, P);
        else if (Dp == 128 && P == 1) store_rows<128, 1, false>(out, bias, tq, rows, Dp, P);
        else if (Dp == 128 && P == 4) store_rows<128, 4, false>(out, bias, tq, rows, Dp, P);
        else if (Dp == 64 && P == 2) store_rows<64, 2, false>(out, bias, tq, rows, Dp, P);
        else if (Dp == 64 && P == 1) store_rows<64, 1, false>(out, bias, tq, rows, Dp, P);
        else if (Dp == 64 && P == 4) store_rows<64, 4, false>(out, bias, tq, rows, Dp, P);
        else store_rows<0, 0, false>(out, bias, tq, rows, Dp, P);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(PSI_FREE + pb));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// bf16 weight images of every head: W_a^T [D_h][D] then W_b^T [D'][D_h]
// (kpiece_img_index), one thread per weight, reads coalesced along the
// fastest index of W_a [D][D_h] and W_b [D_h][D'].
__global__ void phi_mlp_image_kernel(const float* __restrict__ Wa, const float* __restrict__ Wb,
                                     __nv_bfloat16* __restrict__ img, int Dh, int Dp) {
  const int h = blockIdx.y;
  const long long na = static_cast<long long>(Dh) * 128, nb = static_cast<long long>(Dh) * Dp;
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  __nv_bfloat16* out = img + static_cast<long long>(h) * (na + nb);
  if (e < na) {
    const int d = static_cast<int>(e / Dh), j = static_cast<int>(e % Dh);
    out[kpiece_img_index(j, d, Dh)] = __float2bfloat16_rn(Wa[h * na + e]);
  } else if (e < na + nb) {
    const long long e2 = e - na;
    const int j = static_cast<int>(e2 / Dp), f = static_cast<int>(e2 % Dp);
    out[na + kpiece_img_index(f, j, Dp)] = __float2bfloat16_rn(Wb[h * nb + e2]);
  }
}

}  // namespace

bool tc_phi_mlp_eligible(const PhiMlpArgs& a) {
  return a.in_bf16 && a.D == kD && a.Dh >= 128 && a.Dh % 128 == 0 && (a.Dp == 64 || a.Dp == 128) &&
         mlp::smem_bytes(a.Dh, a.Dp) <= mlp::kMaxSmem &&
         (reinterpret_cast<uintptr_t>(a.x) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(a.ba) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(a.bb) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(a.phi) & 15) == 0 && encode_fn() != nullptr;
}

size_t phi_mlp_image_bytes(int heads, int Dh, int Dp) {
  return static_cast<size_t>(heads) * mlp::w_bytes(Dh, Dp);
}

cudaError_t launch_phi_mlp_tc(const PhiMlpArgs& a, void* images, cudaStream_t s) {
  const long long nw = static_cast<long long>(a.Dh) * (128 + a.Dp);
  phi_mlp_image_kernel<<<dim3(static_cast<unsigned>((nw + 255) / 256), a.heads), 256, 0, s>>>(
      a.Wa, a.Wb, static_cast<__nv_bfloat16*>(images), a.Dh, a.Dp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap xmap;
  if (!make_map(&xmap, a.x, a.N, a.BH)) return cudaErrorInvalidValue;
  mlp::Args m;
  m.img = static_cast<const __nv_bfloat16*>(images);
  m.ba = a.ba;
  m.bb = a.bb;
  m.phi = a.phi;
  m.phi_bf16 = a.phi_bf16;
  m.N = a.N;
  m.batch = a.BH / a.heads;
  m.heads = a.heads;
  m.Dh = a.Dh;
  m.Dp = a.Dp;
  m.parts = a.parts;
  m.ntile = static_cast<int>((a.N + 127) / 128);
  const int total = a.BH * m.ntile;
  const int sms = sm_count();
  m.tiles_per_cta = (total + sms - 1) / sms;
  const int ctas = (total + m.tiles_per_cta - 1) / m.tiles_per_cta;
  e = ensure_smem(tc_phi_mlp_kernel, 4, mlp::kMaxSmem);
  if (e != cudaSuccess) return e;
  tc_phi_mlp_kernel<<<ctas, mlp::kThreads, mlp::smem_bytes(a.Dh, a.Dp), s>>>(xmap, m);
  return cudaGetLastError();
}

}  // namespace rehyat

// The feature-map backward's tensor-core passes share this unit too.
#include "tc_phi_bwd.cuh"
