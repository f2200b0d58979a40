// Tensor-core passes of the feature-map backward (bf16 inputs, D = D' = 128).
//
// Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
// Transformers" (papernotes.org note), Method, Key designs 1-5.  With
// g = dL/dy and den = n^S + n^L, through phi = [(x W_1 + b_1)^2, (x W_2 + b_2)^2]
// (u = x W + b, du = 2 u * dphi):
//   q pass, per query row i of chunk t:  dphi_q = (S_L,t g_i - z_L,t (g_i . y_i)) / den_i;
//     dW_q += q^T du_q, db_q += du_q, G_t += phi_q^T (g / den), h_t -= phi_q (g . y) / den;
//   k pass, per key row j of slice s:    dphi_k = Ghat_s v_j + hhat_s;
//     dW_k += k^T du_k, db_k += du_k.
// One CTA per row range (the CUDA-core passes' split and partial layout, so
// their Ghat and reduction passes follow unchanged).  Per 128-row tile:
//   U = X W^T and T = E M^T on tcgen05 (X = q or k tile by TMA; E = g / den
//   built by the converter warps (q pass) or the v tile by TMA (k pass);
//   M = S_L (q) or Ghat (k) converted to bf16 once per CTA), then the
//   converter warps (thread = row) form phi and du from U and T in TMEM and
//   write them to shared memory as bf16, and dW += X^T du (and G += phi^T E)
//   accumulate in TMEM across the CTA's tiles.  The sums over rows of du and
//   phi (g . y) / den come from a warp transpose-reduction (lane l ends with
//   column l of a 32-column chunk).
// Every shared operand tile is [128 rows][128 columns] bf16 in two 64-column
// boxes with the 128-byte swizzle: read K-major (U, T: K = the columns) or
// MN-major (dW, G: K = the rows).
//
// Roles (192 threads): warps 0-3 build E, convert, and write the partials;
// warp 4 TMA producer; warp 5 MMA issuer and TMEM owner.
// TMEM: U [0,128), T [128,256), dW [256,384), G [384,512).

namespace rehyat {
namespace {

namespace pb {
constexpr int kThreads = 192;
constexpr uint32_t kWOff = 0, kMOff = 32768, kXOff = 65536, kEOff = 98304, kDUOff = 131072,
                   kPhiOff = 163840, kVecOff = 196608, kRedOff = 197632, kBarOff = 201728;
enum { W_FULL = 0, M_READY = 1, X_FULL = 2, E_READY = 3, UT_FULL = 4, DU_READY = 5,
       TILE_DONE = 6, DX_FREE = 7, NBAR = 8 };
constexpr uint32_t kSmemBytes = kBarOff + 128 + 1024;
constexpr uint32_t kColU = 0, kColT = 128, kColW = 256, kColG = 384;

// Byte offset of element (row, col) of a [128][128] bf16 tile in two
// 64-column boxes with the 128-byte swizzle (16-byte chunk c of row r at
// c ^ (r mod 8)).
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
  return static_cast<uint32_t>((col >> 6) * 16384 + row * 128 +
                               ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2);
}

// Sum over the warp's 32 lanes of v[i] for each of 32 columns i: lane l
// returns the total of column l (five butterfly stages, 31 shuffles).
__device__ __forceinline__ float transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int m = 16, L = 32; m >= 1; m >>= 1, L >>= 1) {
    const bool hi = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < L / 2; ++i) {
      const float send = hi ? v[i] : v[i + L / 2];
      const float keep = hi ? v[i + L / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  return v[0];
}
}  // namespace pb

struct BwdMaps {
  CUtensorMap x, v;
};

template <bool kQ>
__global__ void __launch_bounds__(pb::kThreads, 1)
    tc_phi_bwd_kernel(const __grid_constant__ BwdMaps maps, const PhiBwdTcArgs a) {
  constexpr uint32_t kWOff = pb::kWOff, kMOff = pb::kMOff, kXOff = pb::kXOff, kEOff = pb::kEOff;
  constexpr uint32_t kDUOff = pb::kDUOff, kPhiOff = pb::kPhiOff;
  using pb::tile_off;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + pb::kBarOff + 8u * i; };
  const uint32_t tmem_slot = pb::kBarOff + 8u * pb::NBAR;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sbase + tmem_slot + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int D = 128, Dp = 128;
  const int bh = blockIdx.z, h = bh % a.heads;
  const long long N = static_cast<long long>(a.T) * a.HW;
  // This CTA's rows: a range of chunk t (q pass) or of slice s (k pass).
  long long r0, r1;
  if (kQ) {
    const int t = blockIdx.y;
    const int first = t * a.Tc, end = min(a.T, first + a.Tc);
    const long long c0 = static_cast<long long>(first) * a.HW, c1 = static_cast<long long>(end) * a.HW;
    const long long span = (c1 - c0 + a.splits - 1) / a.splits;
    r0 = c0 + blockIdx.x * span;
    r1 = min(c1, r0 + span);
  } else {
    const int s = blockIdx.y;
    const long long span = (a.HW + a.splits - 1) / a.splits;
    r0 = static_cast<long long>(s) * a.HW + blockIdx.x * span;
    r1 = min(static_cast<long long>(s + 1) * a.HW, r0 + span);
  }
  const int ntiles = r1 > r0 ? static_cast<int>((r1 - r0 + 127) / 128) : 0;
  const long long set = kQ ? (static_cast<long long>(bh) * a.nchunks + blockIdx.y)
                           : (static_cast<long long>(bh) * a.T + blockIdx.y);
  float* out = a.part + (set * a.splits + blockIdx.x) * (kQ ? 2LL * D * 128 + 256 : 1LL * D * 128 + 128);
  // M (S_L of the chunk, or Ghat of the slice) and its vector (z_L or hhat).
  const float* Msrc = kQ ? a.M + set * Dp * D : a.M + set * (128LL * D + 128);
  const float* vsrc = kQ ? a.vec + set * Dp : Msrc + 128LL * D;
  const bool with_dx = a.dx != nullptr;

  if (tid == 0) {
    for (int i = 0; i < pb::NBAR; ++i) {
      const bool by_rows = i == pb::M_READY || i == pb::DU_READY || (kQ && i == pb::E_READY) ||
                           i == pb::DX_FREE;
      mbar_init(bar(i), by_rows ? 128 : 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     base + tmem_slot),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + tmem_slot);
  float* bvec = reinterpret_cast<float*>(sbase + pb::kVecOff);  // b (128), z_L or hhat (128)
  float* red = reinterpret_cast<float*>(sbase + pb::kRedOff);   // [4 warps][2][128]

  if (warp == 4) {
    // ================================================= TMA producer
    if (lane == 0) {
      bool ok = true;
      // M (S_L of the chunk, or the Ghat block of the slice: contiguous) into
      // L2 for the row warps converting it.
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(Msrc),
                   "r"(static_cast<uint32_t>(kQ ? Dp * D * 4 : (128 * D + 128) * 4))
                   : "memory");
      mbar_expect_tx(bar(pb::W_FULL), Dp * D * 2);
      bulk_load(base + kWOff, static_cast<const uint8_t*>(a.w_img) + static_cast<long long>(h) * Dp * D * 2,
                Dp * D * 2, bar(pb::W_FULL));
      for (int tl = 0; tl < ntiles && ok; ++tl) {
        if (tl > 0) ok = mbar_wait(bar(pb::TILE_DONE), (tl - 1) & 1, abort_flag, 50);
        if (!ok) break;
        const int row = static_cast<int>(r0 + 128LL * tl);
        mbar_expect_tx(bar(pb::X_FULL), kQ ? 32768 : 65536);
        tma_load_3d(base + kXOff, &maps.x, bar(pb::X_FULL), 0, row, bh);
        tma_load_3d(base + kXOff + 16384, &maps.x, bar(pb::X_FULL), 64, row, bh);
        if (kQ && tl + 1 < ntiles) {
          // The next tile's g and y rows (contiguous, 512 bytes a row) into L2
          // for the row warps that build E from them.
          const long long nr0 = r0 + 128LL * (tl + 1);
          const long long nrows = min(128LL, r1 - nr0);
          const uint32_t bytes = static_cast<uint32_t>(nrows) * D * 4;
          const long long gi = (static_cast<long long>(bh) * N + nr0) * D;
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.dy + gi), "r"(bytes)
                       : "memory");
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.y + gi), "r"(bytes)
                       : "memory");
        }
        if (!kQ) {
          tma_load_3d(base + kEOff, &maps.v, bar(pb::X_FULL), 0, row, bh);
          tma_load_3d(base + kEOff + 16384, &maps.v, bar(pb::X_FULL), 64, row, bh);
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ================================================= MMA issuer
    if (lane == 0) {
      const uint32_t id_k = idesc(128, 128, 1, false);          // A, B K-major
      const uint32_t id_mn = idesc_ab(128, 128, 1, true, true);  // A, B MN-major
      const uint32_t id_kmn = idesc(128, 128, 1, true);          // A K-major, B MN-major
      bool ok = mbar_wait(bar(pb::W_FULL), 0, abort_flag, 51) &&
                mbar_wait(bar(pb::M_READY), 0, abort_flag, 52);
      for (int tl = 0; tl < ntiles && ok; ++tl) {
        ok = mbar_wait(bar(pb::X_FULL), tl & 1, abort_flag, 53);
        if (ok && kQ) ok = mbar_wait(bar(pb::E_READY), tl & 1, abort_flag, 54);
        // U's columns hold the previous tile's token gradient until the row
        // warps have read it.
        if (ok && with_dx && tl > 0) ok = mbar_wait(bar(pb::DX_FREE), (tl - 1) & 1, abort_flag, 59);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16(tmem + pb::kColU, sdesc(base + kXOff + off, 16, 1024),
                   sdesc(base + kWOff + off, 16, 1024), id_k, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16(tmem + pb::kColT, sdesc(base + kEOff + off, 16, 1024),
                   sdesc(base + kMOff + off, 16, 1024), id_k, kk > 0);
        }
        mma_commit(bar(pb::UT_FULL));
        ok = mbar_wait(bar(pb::DU_READY), tl & 1, abort_flag, 55);
        if (!ok) break;
        tc_fence_after();
        // dW += X^T du and G += phi^T E: K = the tile's rows, 16 per step.
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = kk * 2048;
          mma_bf16(tmem + pb::kColW, sdesc(base + kXOff + off, 16384, 1024),
                   sdesc(base + kDUOff + off, 16384, 1024), id_mn, (tl > 0 || kk > 0) ? 1u : 0u);
        }
        if (kQ) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = kk * 2048;
            mma_bf16(tmem + pb::kColG, sdesc(base + kPhiOff + off, 16384, 1024),
                     sdesc(base + kEOff + off, 16384, 1024), id_mn, (tl > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (with_dx) {
          // Token gradient through phi: dx = du W (A = du K-major, B = the W
          // image [f][d] read MN-major), into U's columns.
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16(tmem + pb::kColU, sdesc(base + kDUOff + off, 16, 1024),
                     sdesc(base + kWOff + kk * 2048, 16384, 1024), id_kmn, kk > 0);
          }
          if (!kQ && a.dv != nullptr) {
            // dv += phi_k Ghat_s (B = the Ghat tile [f][d] read MN-major),
            // into G's columns (unused by the k pass).
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
              mma_bf16(tmem + pb::kColG, sdesc(base + kPhiOff + off, 16, 1024),
                       sdesc(base + kMOff + kk * 2048, 16384, 1024), id_kmn, kk > 0);
            }
          }
        }
        mma_commit(bar(pb::TILE_DONE));
      }
    }
    __syncwarp();
  } else {
    // ================================================= rows: E, phi, du; partials
    const int r = tid;  // row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    auto wait_all = [&](uint32_t b, uint32_t parity, uint32_t code) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, code));
    };
    bool ok = true;
    // Once per CTA: b, the vector (z_L or hhat), and M as a bf16 K-major
    // operand [f][d] (thread r converts feature row r).
    bvec[r] = __ldg(a.b + static_cast<long long>(h) * Dp + r);
    bvec[128 + r] = __ldg(vsrc + r);
#pragma unroll 4
    for (int d0 = 0; d0 < D; d0 += 8) {
      float m[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        m[i] = kQ ? __ldg(Msrc + sl_index(r, d0 + i, D, Dp)) : __ldg(Msrc + r * D + d0 + i);
      st_shared_v4(base + kMOff + tile_off(r, d0), pack_bf16(m[0], m[1]), pack_bf16(m[2], m[3]),
                   pack_bf16(m[4], m[5]), pack_bf16(m[6], m[7]));
    }
    fence_proxy_async();
    mbar_arrive(bar(pb::M_READY));
    __syncwarp();
    float acc_db[4] = {0.f, 0.f, 0.f, 0.f}, acc_h[4] = {0.f, 0.f, 0.f, 0.f};
    // Adds tile tl's token gradients (in U's and G's columns once TILE_DONE)
    // to dx and dv, then frees the columns for the next tile's U.
    auto flush_dx = [&](int tl) {
      const long long row = r0 + 128LL * tl + r;
      const long long gi = (static_cast<long long>(bh) * N + row) * D;
      const bool with_dv = !kQ && a.dv != nullptr;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rx[32], rv[32];
        REHYAT_TMEM_LD32(lane_base + pb::kColU + c * 32, rx);
        if (with_dv) REHYAT_TMEM_LD32(lane_base + pb::kColG + c * 32, rv);
        tmem_wait_ld();
        if (row < r1) {
          float4* dx4 = reinterpret_cast<float4*>(a.dx + gi + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 o = dx4[i];
            o.x += __uint_as_float(rx[4 * i]);
            o.y += __uint_as_float(rx[4 * i + 1]);
            o.z += __uint_as_float(rx[4 * i + 2]);
            o.w += __uint_as_float(rx[4 * i + 3]);
            dx4[i] = o;
          }
          if (with_dv) {
            float4* dv4 = reinterpret_cast<float4*>(a.dv + gi + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 o = dv4[i];
              o.x += __uint_as_float(rv[4 * i]);
              o.y += __uint_as_float(rv[4 * i + 1]);
              o.z += __uint_as_float(rv[4 * i + 2]);
              o.w += __uint_as_float(rv[4 * i + 3]);
              dv4[i] = o;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(pb::DX_FREE));
    };
    for (int tl = 0; tl < ntiles && ok; ++tl) {
      const long long row = r0 + 128LL * tl + r;
      const bool valid = row < r1;
      float rdot = 0.f;  // (g . y) / den of this row (q pass)
      if (with_dx && tl > 0) {
        ok = wait_all(bar(pb::TILE_DONE), (tl - 1) & 1, 56);
        if (!ok) break;
        tc_fence_after();
        flush_dx(tl - 1);
      }
      if (kQ) {
        // E = g / den for the tile, once the previous tile's MMAs are done.
        if (tl > 0 && !with_dx) ok = wait_all(bar(pb::TILE_DONE), (tl - 1) & 1, 56);
        if (!ok) break;
        const long long gi = (static_cast<long long>(bh) * N + row) * D;
        const float inv = valid ? 1.f / __ldg(a.den + static_cast<long long>(bh) * N + row) : 0.f;
#pragma unroll 2
        for (int d0 = 0; d0 < D; d0 += 8) {
          float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, y0 = g0, y1 = g0;
          if (valid) {
            g0 = __ldg(reinterpret_cast<const float4*>(a.dy + gi + d0));
            g1 = __ldg(reinterpret_cast<const float4*>(a.dy + gi + d0 + 4));
            y0 = __ldg(reinterpret_cast<const float4*>(a.y + gi + d0));
            y1 = __ldg(reinterpret_cast<const float4*>(a.y + gi + d0 + 4));
          }
          rdot += g0.x * y0.x + g0.y * y0.y + g0.z * y0.z + g0.w * y0.w + g1.x * y1.x +
                  g1.y * y1.y + g1.z * y1.z + g1.w * y1.w;
          st_shared_v4(base + kEOff + tile_off(r, d0), pack_bf16(g0.x * inv, g0.y * inv),
                       pack_bf16(g0.z * inv, g0.w * inv), pack_bf16(g1.x * inv, g1.y * inv),
                       pack_bf16(g1.z * inv, g1.w * inv));
        }
        rdot *= inv;
        fence_proxy_async();
        mbar_arrive(bar(pb::E_READY));
      }
      ok = wait_all(bar(pb::UT_FULL), tl & 1, 57);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t ru[32], rt[32];
        REHYAT_TMEM_LD32(lane_base + pb::kColU + c * 32, ru);
        REHYAT_TMEM_LD32(lane_base + pb::kColT + c * 32, rt);
        REHYAT_TMEM_WAIT_LD32(ru);
        REHYAT_TMEM_WAIT_LD32(rt);
        float du[32], ph[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int f = c * 32 + i;
          const float u = __uint_as_float(ru[i]) + bvec[f];
          const float t = __uint_as_float(rt[i]);
          const float dphi = kQ ? t - rdot * bvec[128 + f] : t + bvec[128 + f];
          du[i] = valid ? 2.f * u * dphi : 0.f;
          ph[i] = valid ? u * u : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          st_shared_v4(base + kDUOff + tile_off(r, c * 32 + 8 * j),
                       pack_bf16(du[8 * j], du[8 * j + 1]), pack_bf16(du[8 * j + 2], du[8 * j + 3]),
                       pack_bf16(du[8 * j + 4], du[8 * j + 5]),
                       pack_bf16(du[8 * j + 6], du[8 * j + 7]));
          if (kQ || (with_dx && a.dv != nullptr))
            st_shared_v4(base + kPhiOff + tile_off(r, c * 32 + 8 * j),
                         pack_bf16(ph[8 * j], ph[8 * j + 1]), pack_bf16(ph[8 * j + 2], ph[8 * j + 3]),
                         pack_bf16(ph[8 * j + 4], ph[8 * j + 5]),
                         pack_bf16(ph[8 * j + 6], ph[8 * j + 7]));
        }
        acc_db[c] += pb::transpose_reduce(du, lane);
        if (kQ) {
#pragma unroll
          for (int i = 0; i < 32; ++i) ph[i] *= rdot;
          acc_h[c] -= pb::transpose_reduce(ph, lane);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(pb::DU_READY));
    }
    // Partials: dW [d][f] (TMEM lane d), db, then G [f][d] (lane f) and h.
    if (ok && ntiles > 0) ok = wait_all(bar(pb::TILE_DONE), (ntiles - 1) & 1, 58);
    if (ok && ntiles > 0) {
      tc_fence_after();
      if (with_dx) flush_dx(ntiles - 1);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t rw[32];
        REHYAT_TMEM_LD32(lane_base + pb::kColW + c * 32, rw);
        REHYAT_TMEM_WAIT_LD32(rw);
        float4* o4 = reinterpret_cast<float4*>(out + r * 128 + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          o4[i] = make_float4(__uint_as_float(rw[4 * i]), __uint_as_float(rw[4 * i + 1]),
                              __uint_as_float(rw[4 * i + 2]), __uint_as_float(rw[4 * i + 3]));
        if (kQ) {
          REHYAT_TMEM_LD32(lane_base + pb::kColG + c * 32, rw);
          REHYAT_TMEM_WAIT_LD32(rw);
          float4* g4 = reinterpret_cast<float4*>(out + D * 128 + 128 + r * D + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            g4[i] = make_float4(__uint_as_float(rw[4 * i]), __uint_as_float(rw[4 * i + 1]),
                                __uint_as_float(rw[4 * i + 2]), __uint_as_float(rw[4 * i + 3]));
        }
      }
    }
    // db and h: each warp's per-column sums, then across the four warps.
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      red[(warp * 2) * 128 + c * 32 + lane] = acc_db[c];
      red[(warp * 2 + 1) * 128 + c * 32 + lane] = acc_h[c];
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (ok) {
      float sdb = 0.f, sh = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        sdb += red[(w * 2) * 128 + r];
        sh += red[(w * 2 + 1) * 128 + r];
      }
      out[D * 128 + r] = ntiles > 0 ? sdb : 0.f;
      if (kQ) out[2 * D * 128 + 128 + r] = ntiles > 0 ? sh : 0.f;
      if (ntiles == 0) {  // an empty range still owns its partial block
        for (int i = 0; i < 128; ++i) out[r * 128 + i] = 0.f;
        if (kQ)
          for (int i = 0; i < D; ++i) out[D * 128 + 128 + r * D + i] = 0.f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace

bool tc_phi_bwd_eligible(int in_bf16, int D, int Dp) {
  return in_bf16 && D == 128 && Dp == 128 && encode_fn() != nullptr;
}

cudaError_t launch_phi_bwd_tc(const PhiBwdTcArgs& a, cudaStream_t s) {
  BwdMaps maps;
  memset(&maps, 0, sizeof(maps));
  const long long N = static_cast<long long>(a.T) * a.HW;
  if (!make_map(&maps.x, a.x, N, a.BH)) return cudaErrorInvalidValue;
  if (!a.q_side && !make_map(&maps.v, a.v, N, a.BH)) return cudaErrorInvalidValue;
  if (a.q_side) {
    const cudaError_t e = ensure_smem(tc_phi_bwd_kernel<true>, 6, pb::kSmemBytes);
    if (e != cudaSuccess) return e;
    tc_phi_bwd_kernel<true><<<dim3(a.splits, a.nchunks, a.BH), pb::kThreads, pb::kSmemBytes, s>>>(
        maps, a);
  } else {
    const cudaError_t e = ensure_smem(tc_phi_bwd_kernel<false>, 7, pb::kSmemBytes);
    if (e != cudaSuccess) return e;
    tc_phi_bwd_kernel<false><<<dim3(a.splits, a.T, a.BH), pb::kThreads, pb::kSmemBytes, s>>>(
        maps, a);
  }
  return cudaGetLastError();
}

}  // namespace rehyat
