// Tensor-core passes of the feature-map backward (bf16 inputs, D = D' = 128).
//
// Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
// Transformers" (papernotes.org note), Method, Key designs 1-5.  With
// g = dL/dy and den = n^S + n^L, through phi = [(x W_1 + b_1)^2, (x W_2 + b_2)^2]
// (u = x W + b, du = 2 u * dphi):
//   q pass, per query row i of chunk t:  dphi_q = S_L,t (g_i / den_i) - z_L,t r_i,
//     r_i = g_i . y_i / den_i;  dW_q += q^T du_q, db_q += du_q,
//     G_t += phi_q^T (g / den), h_t -= phi_q r;
//   k pass, per key row j of slice s:    dphi_k = Ghat_s v_j + hhat_s;
//     dW_k += k^T du_k, db_k += du_k.
// One CTA per row range (the CUDA-core passes' split and partial layout for
// dW, db and h; the G blocks are written transposed, [d][f], and the k pass
// reads its Ghat block that way).
//
// Feature orientation: every product puts the 128 features on the TMEM
// lanes and the tile's 128 rows on the columns, so one converter thread owns
// one feature and sums db and h itself.  Per 128-row tile:
//   U^T = W X^T and T^T = M E^T on tcgen05 (A = W or M, [f][d] bf16 in shared
//     memory; B = the X tile (q or k) or E (g / den, from the caller's bf16
//     copy, or the v tile) by TMA);
//   the converter threads read U^T, T^T, form du and phi for their feature
//     over their 64 rows, and write them back over U^T and T^T as bf16 pairs;
//   dW^T += du^T X and G += phi^T E with du^T, phi^T as TMEM A operands and
//     X, E read MN-major from shared memory.
// X and E are double-buffered (the TMA loads tile t + 1 while tile t runs).
// With the token gradients (full backward) du^T and phi^T also go to shared
// memory as [f][rows] tiles (in the second stage's space, so one stage),
// dx^T = W^T du^T lands in U^T's columns and, in the k pass, dv^T =
// Ghat^T phi^T in G's; lane d holds dimension d of 128 rows, so writing dx
// and dv (plain stores: these passes run before the softmax branch's
// kernels, which add their parts) is one 128-byte row segment per warp
// instruction.
//
// Roles (320 threads): warps 0-7 convert, two per TMEM lane quarter: warp w
// owns features 32 (w mod 4) .. + 31 and the tile's rows [64 hf, 64 hf + 64),
// hf = w div 4; warp 8 TMA producer; warp 9 MMA issuer and TMEM owner.
// TMEM: U^T [0,128), T^T [128,256), dW^T [256,384), G [384,512).

namespace rehyat {
namespace {

namespace pb {
constexpr int kThreads = 320;
constexpr int kRowThreads = 256;
constexpr int kTmaWarp = 8, kMmaWarp = 9;
// Shared memory (offsets from a 1024-aligned base): W and M as [f][d] bf16
// tiles, then two stages of (X, E); with token gradients the second stage's
// space holds du^T and phi^T.  Every tile is [128][128] bf16 in two 64-column
// boxes with the 128-byte swizzle.
constexpr uint32_t kWOff = 0, kMOff = 32768, kStage0 = 65536, kStage1 = 131072;
constexpr uint32_t kXRel = 0, kERel = 32768;
constexpr uint32_t kDUOff = kStage1, kPhiOff = kStage1 + 32768;
constexpr uint32_t kVecOff = 196608;          // b (128 floats), z_L or hhat (128)
constexpr uint32_t kRsOff = kVecOff + 1024;   // r of the tile's rows, two tiles [2][128]
constexpr uint32_t kRedOff = kRsOff + 1024;   // [2 halves][2][128] floats
constexpr uint32_t kBarOff = kRedOff + 2048;
enum { W_FULL = 0, M_READY = 1, X_FULL = 2, X_FREE = 4, UT_FULL = 6, DU_READY = 7,
       TILE_DONE = 8, DX_FREE = 9, RS_READY = 10, M_LOAD = 11, NBAR = 12 };
constexpr uint32_t kSmemBytes = kBarOff + 128 + 1024;
constexpr uint32_t kColU = 0, kColT = 128, kColW = 256, kColG = 384;

// Byte offset of element (row, col) of a [128][128] bf16 tile in two
// 64-column boxes with the 128-byte swizzle (16-byte chunk c of row r at
// c ^ (r mod 8)).
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
  return static_cast<uint32_t>((col >> 6) * 16384 + row * 128 +
                               ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2);
}
}  // namespace pb

struct BwdMaps {
  CUtensorMap x, e;
};

template <bool kQ>
__global__ void __launch_bounds__(pb::kThreads, 1)
    tc_phi_bwd_kernel(const __grid_constant__ BwdMaps maps, const PhiBwdTcArgs a) {
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
  // M (S_L of the chunk in the image layout, or the Ghat^T block [d][f] of
  // the slice) and its vector (z_L or hhat).
  const float* Msrc = kQ ? a.M + set * Dp * D : a.M + set * (128LL * D + 128);
  const float* vsrc = kQ ? a.vec + set * Dp : Msrc + 128LL * D;
  const bool with_dx = a.dx != nullptr;
  const bool with_dv = !kQ && with_dx && a.dv != nullptr;
  const int nstage = with_dx ? 1 : 2;
  auto stage_base = [&](int tl) { return base + ((nstage == 2 && (tl & 1)) ? pb::kStage1 : pb::kStage0); };

  if (tid == 0) {
    for (int i = 0; i < pb::NBAR; ++i) {
      const bool by_rows = i == pb::M_READY || i == pb::DU_READY || i == pb::DX_FREE ||
                           i == pb::RS_READY;
      mbar_init(bar(i), by_rows ? pb::kRowThreads : 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == pb::kMmaWarp) {
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
  float* rs = reinterpret_cast<float*>(sbase + pb::kRsOff);     // [2 tiles][128 rows]
  float* red = reinterpret_cast<float*>(sbase + pb::kRedOff);   // [2 halves][2][128]

  if (warp == pb::kTmaWarp) {
    // ================================================= TMA producer
    if (lane == 0) {
      bool ok = true;
      // M in fp32 (64 KB, contiguous) into the second stage's space, where
      // the converters turn it into the bf16 operand before that stage's
      // first tile loads.
      mbar_expect_tx(bar(pb::M_LOAD), Dp * D * 4);
      bulk_load(base + pb::kStage1, Msrc, Dp * D * 4, bar(pb::M_LOAD));
      mbar_expect_tx(bar(pb::W_FULL), Dp * D * 2);
      bulk_load(base + pb::kWOff,
                static_cast<const uint8_t*>(a.w_img) + static_cast<long long>(h) * Dp * D * 2,
                Dp * D * 2, bar(pb::W_FULL));
      for (int tl = 0; tl < ntiles && ok; ++tl) {
        const int st = nstage == 2 ? (tl & 1) : 0;
        if (tl >= nstage) ok = mbar_wait(bar(pb::X_FREE + st), ((tl - nstage) / nstage) & 1, abort_flag, 50);
        // The second stage's first tile waits for the fp32 M to be converted.
        if (ok && nstage == 2 && tl == 1) ok = mbar_wait(bar(pb::M_READY), 0, abort_flag, 48);
        if (!ok) break;
        const int row = static_cast<int>(r0 + 128LL * tl);
        const uint32_t sb = stage_base(tl);
        mbar_expect_tx(bar(pb::X_FULL + st), 65536);
        tma_load_3d(sb + pb::kXRel, &maps.x, bar(pb::X_FULL + st), 0, row, bh);
        tma_load_3d(sb + pb::kXRel + 16384, &maps.x, bar(pb::X_FULL + st), 64, row, bh);
        tma_load_3d(sb + pb::kERel, &maps.e, bar(pb::X_FULL + st), 0, row, bh);
        tma_load_3d(sb + pb::kERel + 16384, &maps.e, bar(pb::X_FULL + st), 64, row, bh);
        if (tl + nstage < ntiles) {
          // The rows of the tile that next uses this stage into L2.
          const long long nr0 = r0 + 128LL * (tl + nstage);
          const uint32_t bytes = static_cast<uint32_t>(min(128LL, r1 - nr0)) * D * 2;
          const long long xi = (static_cast<long long>(bh) * N + nr0) * D * 2;
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                           static_cast<const uint8_t*>(a.x) + xi), "r"(bytes)
                       : "memory");
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                           static_cast<const uint8_t*>(kQ ? a.gh : a.v) + xi), "r"(bytes)
                       : "memory");
        }
      }
    }
    __syncwarp();
  } else if (warp == pb::kMmaWarp) {
    // ================================================= MMA issuer
    if (lane == 0) {
      const uint32_t id_k = idesc(128, 128, 1, false);           // A, B K-major
      const uint32_t id_kmn = idesc(128, 128, 1, true);          // B MN-major (A from TMEM)
      const uint32_t id_mn = idesc_ab(128, 128, 1, true, true);  // A, B MN-major
      bool ok = mbar_wait(bar(pb::W_FULL), 0, abort_flag, 51) &&
                mbar_wait(bar(pb::M_READY), 0, abort_flag, 52);
      for (int tl = 0; tl < ntiles && ok; ++tl) {
        const int st = nstage == 2 ? (tl & 1) : 0;
        const uint32_t sb = stage_base(tl);
        ok = mbar_wait(bar(pb::X_FULL + st), (tl / nstage) & 1, abort_flag, 53);
        // U^T's columns hold the previous tile's dx^T until the converter
        // threads have read it.
        if (ok && with_dx && tl > 0) ok = mbar_wait(bar(pb::DX_FREE), (tl - 1) & 1, abort_flag, 59);
        if (!ok) break;
        tc_fence_after();
        mma8_ss_kmajor(tmem + pb::kColU, sdesc(base + pb::kWOff, 16, 1024),
                       sdesc(sb + pb::kXRel, 16, 1024), id_k, 0u);
        mma8_ss_kmajor(tmem + pb::kColT, sdesc(base + pb::kMOff, 16, 1024),
                       sdesc(sb + pb::kERel, 16, 1024), id_k, 0u);
        mma_commit(bar(pb::UT_FULL));
        ok = mbar_wait(bar(pb::DU_READY), tl & 1, abort_flag, 55);
        if (!ok) break;
        tc_fence_after();
        // dW^T += du^T X and G += phi^T E: A from TMEM (the two halves' rows
        // in two runs of columns), K = the tile's rows, 16 per step.
        mma8_ts_mn_split(tmem + pb::kColW, tmem + pb::kColU, sdesc(sb + pb::kXRel, 16384, 1024),
                         id_kmn, tl > 0 ? 1u : 0u);
        if (kQ)
          mma8_ts_mn_split(tmem + pb::kColG, tmem + pb::kColT, sdesc(sb + pb::kERel, 16384, 1024),
                           id_kmn, tl > 0 ? 1u : 0u);
        // The stage's X and E are read by nothing after these: the TMA may
        // refill it while the token-gradient products below run.
        mma_commit(bar(pb::X_FREE + st));
        if (with_dx) {
          // dx^T = W^T du^T (A = W read MN-major, B = du^T [f][rows]) into
          // U^T's columns, after the products above have read them.
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + pb::kColU, sdesc(base + pb::kWOff + kk * 2048, 16384, 1024),
                     sdesc(base + pb::kDUOff + kk * 2048, 16384, 1024), id_mn, kk > 0);
          if (with_dv) {
            // dv^T = Ghat^T phi^T (A = the Ghat tile read MN-major) into G's
            // columns, unused by the k pass.
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_bf16(tmem + pb::kColG, sdesc(base + pb::kMOff + kk * 2048, 16384, 1024),
                       sdesc(base + pb::kPhiOff + kk * 2048, 16384, 1024), id_mn, kk > 0);
          }
        }
        mma_commit(bar(pb::TILE_DONE));
      }
    }
    __syncwarp();
  } else {
    // ================================================= converters
    const int f = tid & 127;   // feature == TMEM lane (dimension d for dx^T, dv^T)
    const int hf = warp >> 2;  // rows [64 hf, 64 hf + 64) of each tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    auto wait_all = [&](uint32_t b, uint32_t parity, uint32_t code) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, code));
    };
    bool ok = true;
    // Once per CTA: b, the vector (z_L or hhat), and M as a bf16 [f][d]
    // tile from its fp32 copy in shared memory; thread (f, hf) converts
    // dimensions [64 hf, 64 hf + 64) of feature f (both sources keep
    // consecutive features contiguous for a fixed d: no bank conflicts).
    if (hf == 0) {
      bvec[f] = __ldg(a.b + static_cast<long long>(h) * Dp + f);
      bvec[128 + f] = __ldg(vsrc + f);
    }
    ok = wait_all(bar(pb::M_LOAD), 0, 47);
    const float* Ms = reinterpret_cast<const float*>(sbase + pb::kStage1);
#pragma unroll 2
    for (int d0 = 64 * hf; d0 < 64 * hf + 64 && ok; d0 += 8) {
      float m[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        m[i] = kQ ? Ms[sl_index(f, d0 + i, D, Dp)] : Ms[(d0 + i) * 128 + f];
      st_shared_v4(base + pb::kMOff + tile_off(f, d0), pack_bf16(m[0], m[1]), pack_bf16(m[2], m[3]),
                   pack_bf16(m[4], m[5]), pack_bf16(m[6], m[7]));
    }
    fence_proxy_async();
    asm volatile("bar.sync 1, %0;" ::"r"(pb::kRowThreads) : "memory");
    mbar_arrive(bar(pb::M_READY));
    const float bf = bvec[f], vf = bvec[128 + f];
    float acc_db = 0.f, acc_h = 0.f;
    // dx^T (U^T's columns, lane d) and dv^T (G's columns) of tile tl written
    // to dx and dv: per row a warp instruction covers 32 consecutive d.
    auto flush_dx = [&](int tl) {
      const long long rowbase = r0 + 128LL * tl;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int j0 = 64 * hf + 32 * c;
        uint32_t rx[32], rv[32];
        REHYAT_TMEM_LD32(lane_base + pb::kColU + j0, rx);
        if (with_dv) REHYAT_TMEM_LD32(lane_base + pb::kColG + j0, rv);
        tmem_wait_ld();
        const int nvalid = static_cast<int>(min(32LL, max(0LL, r1 - (rowbase + j0))));
        float* dxr = a.dx + (static_cast<long long>(bh) * N + rowbase + j0) * D + f;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i < nvalid) dxr[static_cast<long long>(i) * D] = __uint_as_float(rx[i]);
        if (with_dv) {
          float* dvr = a.dv + (static_cast<long long>(bh) * N + rowbase + j0) * D + f;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nvalid) dvr[static_cast<long long>(i) * D] = __uint_as_float(rv[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(pb::DX_FREE));
    };
    for (int tl = 0; tl < ntiles && ok; ++tl) {
      const long long rowbase = r0 + 128LL * tl;
      const float* rt_rows = rs + (tl & 1) * 128;
      if (kQ) {
        // r of the tile's rows, shared by every feature.
        if (hf == 0) {
          const long long row = rowbase + f;
          rs[(tl & 1) * 128 + f] = row < r1 ? __ldg(a.r + static_cast<long long>(bh) * N + row) : 0.f;
        }
        mbar_arrive(bar(pb::RS_READY));
        ok = wait_all(bar(pb::RS_READY), tl & 1, 49);
        if (!ok) break;
      }
      ok = wait_all(bar(pb::UT_FULL), tl & 1, 57);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int j0 = 64 * hf + 32 * c;  // the chunk's first row in the tile
        uint32_t ru[32], rt[32];
        REHYAT_TMEM_LD32(lane_base + pb::kColU + j0, ru);
        REHYAT_TMEM_LD32(lane_base + pb::kColT + j0, rt);
        REHYAT_TMEM_WAIT_LD32(ru);
        REHYAT_TMEM_WAIT_LD32(rt);
        const int nvalid = static_cast<int>(min(32LL, max(0LL, r1 - (rowbase + j0))));
        uint32_t pdu[16], pph[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float du2[2], ph2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float u = __uint_as_float(ru[i + e]) + bf;
            const float t = __uint_as_float(rt[i + e]);
            const float rr = kQ ? rt_rows[j0 + i + e] : 0.f;
            const float dphi = kQ ? t - rr * vf : t + vf;
            const bool valid = i + e < nvalid;
            du2[e] = valid ? 2.f * u * dphi : 0.f;
            ph2[e] = valid ? u * u : 0.f;
            acc_db += du2[e];
            if (kQ) acc_h = fmaf(-ph2[e], rr, acc_h);
          }
          pdu[i / 2] = pack_bf16(du2[0], du2[1]);
          pph[i / 2] = pack_bf16(ph2[0], ph2[1]);
        }
        // du^T and phi^T as bf16 row pairs over the columns this chunk has
        // read: rows [j0, j0 + 32) go to columns [64 hf + 16 c, + 16).
        REHYAT_TMEM_ST16(lane_base + pb::kColU + 64 * hf + 16 * c, pdu);
        REHYAT_TMEM_ST16(lane_base + pb::kColT + 64 * hf + 16 * c, pph);
        if (with_dx) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            st_shared_v4(base + pb::kDUOff + tile_off(f, j0 + 8 * j), pdu[4 * j], pdu[4 * j + 1],
                         pdu[4 * j + 2], pdu[4 * j + 3]);
            if (with_dv)
              st_shared_v4(base + pb::kPhiOff + tile_off(f, j0 + 8 * j), pph[4 * j],
                           pph[4 * j + 1], pph[4 * j + 2], pph[4 * j + 3]);
          }
        }
      }
      tmem_wait_st();
      if (with_dx) fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(pb::DU_READY));
      if (with_dx) {
        ok = wait_all(bar(pb::TILE_DONE), tl & 1, 56);
        if (!ok) break;
        tc_fence_after();
        flush_dx(tl);
      }
    }
    // Partials: dW^T lane f -> dW [d][f], G lane f -> G^T [d][f]: for a fixed
    // d a warp writes 32 consecutive floats.  Then db and h (the two halves'
    // sums in order).
    if (ok && ntiles > 0 && !with_dx) ok = wait_all(bar(pb::TILE_DONE), (ntiles - 1) & 1, 58);
    if (ok && ntiles > 0) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 2 * hf; c < 2 * hf + 2; ++c) {
        uint32_t rw[32];
        REHYAT_TMEM_LD32(lane_base + pb::kColW + c * 32, rw);
        REHYAT_TMEM_WAIT_LD32(rw);
#pragma unroll
        for (int i = 0; i < 32; ++i) out[(c * 32 + i) * 128 + f] = __uint_as_float(rw[i]);
        if (kQ) {
          REHYAT_TMEM_LD32(lane_base + pb::kColG + c * 32, rw);
          REHYAT_TMEM_WAIT_LD32(rw);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            out[D * 128 + 128 + (c * 32 + i) * 128 + f] = __uint_as_float(rw[i]);
        }
      }
    }
    red[(hf * 2) * 128 + f] = acc_db;
    red[(hf * 2 + 1) * 128 + f] = acc_h;
    asm volatile("bar.sync 1, %0;" ::"r"(pb::kRowThreads) : "memory");
    if (ok && hf == 0) {
      out[D * 128 + f] = ntiles > 0 ? red[f] + red[2 * 128 + f] : 0.f;
      if (kQ) out[2 * D * 128 + 128 + f] = ntiles > 0 ? red[128 + f] + red[3 * 128 + f] : 0.f;
    }
    if (ok && ntiles == 0) {  // an empty range still owns its partial block
      for (int i = 64 * hf; i < 64 * hf + 64; ++i) out[i * 128 + f] = 0.f;
      if (kQ)
        for (int i = 64 * hf; i < 64 * hf + 64; ++i) out[D * 128 + 128 + i * 128 + f] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == pb::kMmaWarp) {
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
  // E: the caller's bf16 g / den (q pass) or v (k pass).
  if (a.q_side && (a.gh == nullptr || a.r == nullptr)) return cudaErrorInvalidValue;
  if (!make_map(&maps.x, a.x, N, a.BH) || !make_map(&maps.e, a.q_side ? a.gh : a.v, N, a.BH))
    return cudaErrorInvalidValue;
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
