// Tensor-core kernels of the full backward's softmax branch (bf16 inputs,
// D = 128): dq (query-parallel) and dk, dv (key-parallel).
//
// Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
// Transformers" (papernotes.org note), Method, Key designs 1-5 (the second
// training stage fine-tunes the whole model, so gradients reach q, k, v).
// For a query i with window W_t, gh_i = g_i / den_i, r_i = (g_i . y_i)/den_i:
//   P_ij = exp(s_ij - c_i),  dS_ij = P_ij (gh_i.v_j - r_i) - [j = j*_i] Dc_i,
//   Dc_i = sum_j P_ij (gh_i.v_j - r_i),
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
//   dv_j = sum_i P_ij gh_i
// (the linear branch's part is added by separate kernels).  j*_i is the key
// with the largest logit as recomputed here (lowest index among equal ones).
//
// dq kernel, per CTA one 128-row query tile of a chunk, streaming the
// window's key tiles:
//   S = Q K^T and dP = GH V^T on tcgen05 (bf16, fp32 in TMEM; GH = bf16 of
//   g / den from the prep pass), S double-buffered so S of tile j + 2 is
//   computed while tile j is converted; eight warps, two per row (columns
//   [64 hf, 64 hf + 64)), form P and dS in fp32 and write dS back into their
//   own columns of S as bf16 pairs, the A operand of dQ += dS K (K read
//   MN-major from the same shared tile that fed S).  Each half keeps its
//   part of Dc and of the arg-max; they are combined through TMEM at the end.
//   Roles (320 threads): warps 0-7 convert + epilogue, warp 8 TMA, warp 9
//   MMA issuer and TMEM owner.  TMEM: S0 [0,128), dP [128,256),
//   dQ [256,384), S1 [384,512).
//
// dk/dv kernel, per CTA one 128-row key tile, streaming the query tiles of
// the chunks whose window holds a key of the tile, in the transposed
// orientation so the products' A operands come straight from TMEM:
//   S^T = K Q^T, dP^T = V GH^T (M = keys); the eight warps (two per key row,
//   query columns [64 hf, 64 hf + 64)) form P^T = exp(s - c_i) and
//   dS^T = P^T (dP^T - r_i) - [j = j*_i] Dc_i with per-column c, r, Dc, j*
//   staged in shared memory, write P^T over S^T and dS^T over dP^T (bf16
//   pairs, own columns), then dV += P^T GH and dK += dS^T Q (GH and Q read
//   MN-major).  TMEM: S^T [0,128), dP^T [128,256), dV [256,384), dK [384,512).
//
// Every wait is bounded (tc_common.cuh); a timeout sets rehyat_tc_error.

namespace rehyat {

namespace {

namespace bq {
constexpr int kThreads = 320;
constexpr uint32_t kQOff = 0, kGOff = 32768, kKOff = 65536;   // Q, GH, K ring (3 x 32 KB)
constexpr uint32_t kVOff = kKOff + 3 * 32768;                   // V ring (2 x 32 KB)
constexpr uint32_t kBarOff = kVOff + 2 * 32768;
enum { QG_FULL = 0, K_FULL = 1, K_EMPTY = 4, V_FULL = 7, V_EMPTY = 9, S_FULL = 11, DP_FULL = 13,
       DS_FULL = 14, DQ_DONE = 15, XCH = 16, NBAR = 17 };
constexpr uint32_t kTmemSlot = kBarOff + 8 * NBAR;
constexpr uint32_t kAbortSlot = kTmemSlot + 4;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kColS0 = 0, kColDP = 128, kColDQ = 256, kColS1 = 384;
}  // namespace bq

struct AttnBwdMaps {
  CUtensorMap q, k, v, gh;
};

__global__ void __launch_bounds__(bq::kThreads, 1)
    tc_bwd_dq_kernel(const __grid_constant__ AttnBwdMaps maps, const AttnBwdTcArgs A) {
  // Local names shadow the forward kernels' constants of the same names.
  constexpr uint32_t kQOff = bq::kQOff, kGOff = bq::kGOff, kKOff = bq::kKOff, kVOff = bq::kVOff;
  constexpr uint32_t kBarOff = bq::kBarOff, kTmemSlot = bq::kTmemSlot, kAbortSlot = bq::kAbortSlot;
  constexpr uint32_t kColS0 = bq::kColS0, kColS1 = bq::kColS1, kColDP = bq::kColDP,
                     kColDQ = bq::kColDQ;
  using bq::QG_FULL;
  using bq::K_FULL;
  using bq::K_EMPTY;
  using bq::V_FULL;
  using bq::V_EMPTY;
  using bq::S_FULL;
  using bq::DP_FULL;
  using bq::DS_FULL;
  using bq::DQ_DONE;
  using bq::XCH;
  using bq::NBAR;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + kBarOff + 8u * i; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sbase + kAbortSlot);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = blockIdx.y, bh = blockIdx.z;
  const int first = t * A.Tc, end = min(A.T, first + A.Tc), w = max(first - A.To, 0);
  const int q_end = end * A.HW;
  const int row0 = first * A.HW + blockIdx.x * 128;
  if (row0 >= q_end) return;
  const int nrows = min(128, q_end - row0);
  const int k0 = w * A.HW, na = q_end - k0;
  const int nt = (na + 127) / 128;
  const long long N = static_cast<long long>(A.T) * A.HW;
  const long long base_row = static_cast<long long>(bh) * N;

  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i)
      mbar_init(bar(i), (i == DS_FULL || i == XCH) ? 256 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     base + kTmemSlot), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + kTmemSlot);

  if (warp == 8) {
    // ================================================= TMA producer
    if (lane == 0) {
      bool ok = true;
      mbar_expect_tx(bar(QG_FULL), 4 * 16384);
      tma_load_3d(base + kQOff, &maps.q, bar(QG_FULL), 0, row0, bh);
      tma_load_3d(base + kQOff + 16384, &maps.q, bar(QG_FULL), 64, row0, bh);
      tma_load_3d(base + kGOff, &maps.gh, bar(QG_FULL), 0, row0, bh);
      tma_load_3d(base + kGOff + 16384, &maps.gh, bar(QG_FULL), 64, row0, bh);
      for (int j = 0; j < nt && ok; ++j) {
        const int row = k0 + j * 128;
        const int ks = j % 3;
        if (j >= 3) ok = mbar_wait(bar(K_EMPTY + ks), ((j - 3) / 3) & 1, abort_flag, 19);
        if (!ok) break;
        mbar_expect_tx(bar(K_FULL + ks), 32768);
        tma_load_3d(base + kKOff + ks * 32768, &maps.k, bar(K_FULL + ks), 0, row, bh);
        tma_load_3d(base + kKOff + ks * 32768 + 16384, &maps.k, bar(K_FULL + ks), 64, row, bh);
        const int vs = j & 1;
        if (j >= 2) ok = mbar_wait(bar(V_EMPTY + vs), ((j - 2) >> 1) & 1, abort_flag, 20);
        if (!ok) break;
        mbar_expect_tx(bar(V_FULL + vs), 32768);
        tma_load_3d(base + kVOff + vs * 32768, &maps.v, bar(V_FULL + vs), 0, row, bh);
        tma_load_3d(base + kVOff + vs * 32768 + 16384, &maps.v, bar(V_FULL + vs), 64, row, bh);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ================================================= MMA issuer
    if (lane == 0) {
      const uint32_t id_kk = idesc(128, 128, 1, false);  // A, B K-major
      const uint32_t id_dq = idesc(128, 128, 1, true);   // B (K tile) MN-major
      bool ok = mbar_wait(bar(QG_FULL), 0, abort_flag, 21);
      auto s_buf = [&](int j) { return tmem + ((j & 1) ? kColS1 : kColS0); };
      // S(j) = Q K(j)^T into S buffer j & 1.
      auto issue_s = [&](int j) -> bool {
        if (!mbar_wait(bar(K_FULL + j % 3), (j / 3) & 1, abort_flag, 22)) return false;
        tc_fence_after();
        const uint32_t kaddr = base + kKOff + (j % 3) * 32768;
        mma8_ss_kmajor(s_buf(j), sdesc(base + kQOff, 16, 1024), sdesc(kaddr, 16, 1024), id_kk, 0u);
        mma_commit(bar(S_FULL + (j & 1)));
        return true;
      };
      // dP(j) = GH V(j)^T.
      auto issue_dp = [&](int j) -> bool {
        if (!mbar_wait(bar(V_FULL + (j & 1)), (j >> 1) & 1, abort_flag, 23)) return false;
        tc_fence_after();
        const uint32_t vaddr = base + kVOff + (j & 1) * 32768;
        mma8_ss_kmajor(tmem + kColDP, sdesc(base + kGOff, 16, 1024), sdesc(vaddr, 16, 1024), id_kk,
                       0u);
        mma_commit(bar(DP_FULL));
        mma_commit(bar(V_EMPTY + (j & 1)));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && nt > 1) ok = issue_s(1);
      if (ok) ok = issue_dp(0);
      for (int j = 0; j < nt && ok; ++j) {
        // dS(j) is in S buffer j & 1 and dP(j) has been read.
        ok = mbar_wait(bar(DS_FULL), j & 1, abort_flag, 24);
        if (!ok) break;
        tc_fence_after();
        if (j + 1 < nt && !(ok = issue_dp(j + 1))) break;
        // dQ += dS(j) K(j): dS of key columns [0, 64) sits in columns [0, 32)
        // of the buffer, of [64, 128) in columns [64, 96) (one run per half).
        const uint32_t kaddr = base + kKOff + (j % 3) * 32768;
        mma8_ts_mn_split(tmem + kColDQ, s_buf(j), sdesc(kaddr, 16384, 1024), id_dq,
                         j > 0 ? 1u : 0u);
        mma_commit(bar(K_EMPTY + j % 3));
        // S(j + 2) overwrites this buffer after dQ(j) has read it (in order).
        if (j + 2 < nt && !(ok = issue_s(j + 2))) break;
      }
      if (ok) mma_commit(bar(DQ_DONE));
    }
    __syncwarp();
  } else {
    // ================================================= convert + epilogue
    const int hf = warp >> 2;
    const int r = tid & 127;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    auto wait_all = [&](uint32_t b, uint32_t parity, uint32_t code) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, code));
    };
    const long long grow = base_row + row0 + r;
    const bool valid = r < nrows;
    constexpr float kLog2e = 1.4426950408889634f;
    const float sl2 = A.scale * kLog2e;
    const float m = valid ? __ldg(A.c + grow) * kLog2e : 0.f;
    const float rr = valid ? __ldg(A.r + grow) : 0.f;
    float Dc = 0.f, best = -INFINITY;
    int barg = 0x7fffffff;
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      const int nvalid = min(128, na - j * 128);
      const uint32_t sb = lane_base + ((j & 1) ? kColS1 : kColS0);
      // Phase 1 (needs S only, so it overlaps dP's MMAs): P of this half's
      // 64 key columns in fp32, and the arg-max.
      ok = wait_all(bar(S_FULL + (j & 1)), (j >> 1) & 1, 25);
      if (!ok) break;
      tc_fence_after();
      float pv[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t xs[32];
        REHYAT_TMEM_LD32(sb + 64 * hf + 32 * c, xs);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = 64 * hf + 32 * c + i;
          const float sv = __uint_as_float(xs[i]);
          float p = 0.f;
          if (key < nvalid) {
            p = ex2(fmaf(sv, sl2, -m));
            if (sv > best) {
              best = sv;
              barg = j * 128 + key;
            }
          }
          pv[32 * c + i] = p;
        }
      }
      // Phase 2: dS = P (dP - r) once dP is done; dS (bf16 pairs) goes over
      // this half's own S columns.
      ok = wait_all(bar(DP_FULL), j & 1, 26);
      if (!ok) break;
      tc_fence_after();
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t xd[32];
        REHYAT_TMEM_LD32(lane_base + kColDP + 64 * hf + 32 * c, xd);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float d0 = pv[32 * c + i] * (__uint_as_float(xd[i]) - rr);
          const float d1 = pv[32 * c + i + 1] * (__uint_as_float(xd[i + 1]) - rr);
          Dc += d0 + d1;
          pk[16 * c + i / 2] = pack_bf16(d0, d1);
        }
      }
      REHYAT_TMEM_ST32(sb + 64 * hf, pk);
      tmem_wait_st();
      if (nvalid < 128 && r >= nvalid) {
        // K rows past the window are zeroed before dQ += dS K reads them
        // (their dS is 0; this keeps 0 * garbage out of dQ).
        const uint32_t krow = base + kKOff + (j % 3) * 32768 + hf * 16384 + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) st_shared_v4(krow + c * 16, 0, 0, 0, 0);
      }
      if (nvalid < 128) fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(DS_FULL));
    }
    // Combine the halves: each writes (Dc, best logit, its key) into TMEM
    // columns of S0 (half 0: 0..2, half 1: 4..6) once every MMA is done.
    if (ok) ok = wait_all(bar(DQ_DONE), 0, 27);
    if (ok) {
      tc_fence_after();
      const uint32_t mine = lane_base + kColS0 + 4 * hf, theirs = lane_base + kColS0 + 4 * (1 - hf);
      tmem_st1(mine, __float_as_uint(Dc));
      tmem_st1(mine + 1, __float_as_uint(best));
      tmem_st1(mine + 2, static_cast<uint32_t>(barg));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(XCH));
      ok = wait_all(bar(XCH), 0, 28);
      if (ok) {
        tc_fence_after();
        const float oDc = __uint_as_float(tmem_ld1(theirs));
        const float obest = __uint_as_float(tmem_ld1(theirs + 1));
        const int oarg = static_cast<int>(tmem_ld1(theirs + 2));
        // Same sums in the same order on both halves: h0 + h1.
        Dc = hf == 0 ? Dc + oDc : oDc + Dc;
        if (obest > best || (obest == best && oarg < barg)) {
          best = obest;
          barg = oarg;
        }
      }
    }
    if (ok) {
      // dq = scale (dQ - Dc k_{j*}); half hf writes columns [64 hf, 64 hf + 64).
      // (No key is found only for rows whose logits are all NaN.)
      const bool has = barg != 0x7fffffff;
      const long long js = base_row + k0 + (has ? barg : 0);
      const __nv_bfloat16* krow = static_cast<const __nv_bfloat16*>(A.k) + js * 128 + 64 * hf;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        REHYAT_TMEM_LD32(lane_base + kColDQ + 64 * hf + 32 * c, o);
        tmem_wait_ld();
        if (valid) {
          float* dst = A.dq + grow * 128 + 64 * hf + 32 * c;
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 v4;
            const uint2 kb = has ? *reinterpret_cast<const uint2*>(krow + 32 * c + i)
                                 : make_uint2(0u, 0u);
            const float k0v = __uint_as_float(kb.x << 16), k1v = __uint_as_float(kb.x & 0xFFFF0000u);
            const float k2v = __uint_as_float(kb.y << 16), k3v = __uint_as_float(kb.y & 0xFFFF0000u);
            v4.x = A.scale * (__uint_as_float(o[i]) - Dc * k0v);
            v4.y = A.scale * (__uint_as_float(o[i + 1]) - Dc * k1v);
            v4.z = A.scale * (__uint_as_float(o[i + 2]) - Dc * k2v);
            v4.w = A.scale * (__uint_as_float(o[i + 3]) - Dc * k3v);
            if (A.accumulate) {  // dq already holds the linear branch's part
              const float4 p4 = *reinterpret_cast<const float4*>(dst + i);
              v4.x += p4.x;
              v4.y += p4.y;
              v4.z += p4.z;
              v4.w += p4.w;
            }
            *reinterpret_cast<float4*>(dst + i) = v4;
          }
        }
      }
      if (valid && hf == 0) {
        A.Dc[grow] = Dc;
        A.jstar[grow] = has ? static_cast<int>(k0 + barg) : -1;
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

namespace bk {
constexpr int kThreads = 320;
constexpr uint32_t kKOff = 0, kVOff = 32768;                 // the CTA's K and V tiles
constexpr uint32_t kQOff = 65536;                            // Q ring (2 x 32 KB)
constexpr uint32_t kGOff = kQOff + 2 * 32768;                // GH ring (2 x 32 KB)
constexpr uint32_t kVecOff = kGOff + 2 * 32768;              // per-query m, r, Dc, j* (2 x 2 KB)
constexpr uint32_t kBarOff = kVecOff + 2 * 2048;
enum { KV_FULL = 0, QG_FULL = 1, QG_EMPTY = 3, VEC_FULL = 5, ST_FULL = 7, DS_FULL = 8,
       KV_DONE = 9, DPT_FULL = 10, PT_FULL = 11, NBAR = 12 };
constexpr uint32_t kTmemSlot = kBarOff + 8 * NBAR;
constexpr uint32_t kAbortSlot = kTmemSlot + 4;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

// The (chunk, 128-row query tile) pairs whose window holds a key of the key
// tile [j0, j1), in chunk order; every role walks the same list.
struct QWalk {
  int T, HW, Tc, To, nchunks, j0, j1;
  int t = 0, qt = 0;
  int first = 0, end = 0, w = 0;
  __device__ bool hits(int tt) const {
    const int f = tt * Tc, e = min(T, f + Tc), ww = max(f - To, 0);
    return ww * HW < j1 && e * HW > j0;
  }
  __device__ void set(int tt) {
    t = tt;
    first = tt * Tc;
    end = min(T, first + Tc);
    w = max(first - To, 0);
    qt = 0;
  }
  // Moves to the first pair at or after chunk tt; false when there is none.
  __device__ bool seek(int tt) {
    while (tt < nchunks && !hits(tt)) ++tt;
    if (tt >= nchunks) return false;
    set(tt);
    return true;
  }
  __device__ bool next() {
    if (first * HW + (qt + 1) * 128 < end * HW) {
      ++qt;
      return true;
    }
    return seek(t + 1);
  }
  __device__ int q0() const { return first * HW + qt * 128; }
  __device__ int qvalid() const { return min(128, end * HW - q0()); }
};
}  // namespace bk

__global__ void __launch_bounds__(bk::kThreads, 1)
    tc_bwd_dkv_kernel(const __grid_constant__ AttnBwdMaps maps, const AttnBwdTcArgs A) {
  constexpr uint32_t kKOff = bk::kKOff, kVOff = bk::kVOff, kQOff = bk::kQOff, kGOff = bk::kGOff;
  constexpr uint32_t kVecOff = bk::kVecOff, kBarOff = bk::kBarOff, kTmemSlot = bk::kTmemSlot,
                     kAbortSlot = bk::kAbortSlot;
  constexpr uint32_t kColS = bk::kColS, kColDP = bk::kColDP, kColDV = bk::kColDV,
                     kColDK = bk::kColDK;
  using bk::KV_FULL;
  using bk::QG_FULL;
  using bk::QG_EMPTY;
  using bk::VEC_FULL;
  using bk::ST_FULL;
  using bk::DS_FULL;
  using bk::KV_DONE;
  using bk::DPT_FULL;
  using bk::PT_FULL;
  using bk::NBAR;
  using bk::QWalk;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + kBarOff + 8u * i; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sbase + kAbortSlot);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int N = A.T * A.HW;
  const int j0 = blockIdx.x * 128;
  if (j0 >= N) return;
  const int j1 = min(N, j0 + 128);
  const long long base_row = static_cast<long long>(bh) * N;
  // Number of (chunk, query tile) pairs.
  int niter = 0;
  {
    QWalk w{A.T, A.HW, A.Tc, A.To, A.nchunks, j0, j1};
    if (w.seek(0))
      do ++niter;
      while (w.next());
  }

  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i)
      mbar_init(bar(i), (i == DS_FULL || i == PT_FULL || i == VEC_FULL || i == VEC_FULL + 1)
                            ? 256 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     base + kTmemSlot), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + kTmemSlot);

  if (warp == 8) {
    // ================================================= TMA producer
    if (lane == 0) {
      bool ok = true;
      mbar_expect_tx(bar(KV_FULL), 4 * 16384);
      tma_load_3d(base + kKOff, &maps.k, bar(KV_FULL), 0, j0, bh);
      tma_load_3d(base + kKOff + 16384, &maps.k, bar(KV_FULL), 64, j0, bh);
      tma_load_3d(base + kVOff, &maps.v, bar(KV_FULL), 0, j0, bh);
      tma_load_3d(base + kVOff + 16384, &maps.v, bar(KV_FULL), 64, j0, bh);
      QWalk w{A.T, A.HW, A.Tc, A.To, A.nchunks, j0, j1};
      w.seek(0);
      for (int i = 0; i < niter && ok; ++i, w.next()) {
        const int st = i & 1;
        if (i >= 2) ok = mbar_wait(bar(QG_EMPTY + st), ((i - 2) >> 1) & 1, abort_flag, 19);
        if (!ok) break;
        mbar_expect_tx(bar(QG_FULL + st), 4 * 16384);
        const uint32_t qd = base + kQOff + st * 32768, gd = base + kGOff + st * 32768;
        tma_load_3d(qd, &maps.q, bar(QG_FULL + st), 0, w.q0(), bh);
        tma_load_3d(qd + 16384, &maps.q, bar(QG_FULL + st), 64, w.q0(), bh);
        tma_load_3d(gd, &maps.gh, bar(QG_FULL + st), 0, w.q0(), bh);
        tma_load_3d(gd + 16384, &maps.gh, bar(QG_FULL + st), 64, w.q0(), bh);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ================================================= MMA issuer
    if (lane == 0) {
      const uint32_t id_kk = idesc(128, 128, 1, false);  // A, B K-major
      const uint32_t id_mn = idesc(128, 128, 1, true);   // B MN-major
      bool ok = mbar_wait(bar(KV_FULL), 0, abort_flag, 21);
      auto qa_of = [&](int i) { return base + kQOff + (i & 1) * 32768; };
      auto ga_of = [&](int i) { return base + kGOff + (i & 1) * 32768; };
      // S^T(i) = K Q(i)^T and dP^T(i) = V GH(i)^T, committed separately so
      // the exponentials can start before dP^T is done.
      auto issue_st = [&](int i) -> bool {
        if (!mbar_wait(bar(QG_FULL + (i & 1)), (i >> 1) & 1, abort_flag, 22)) return false;
        tc_fence_after();
        mma8_ss_kmajor(tmem + kColS, sdesc(base + kKOff, 16, 1024), sdesc(qa_of(i), 16, 1024),
                       id_kk, 0u);
        mma_commit(bar(ST_FULL));
        return true;
      };
      auto issue_dpt = [&](int i) {
        mma8_ss_kmajor(tmem + kColDP, sdesc(base + kVOff, 16, 1024), sdesc(ga_of(i), 16, 1024),
                       id_kk, 0u);
        mma_commit(bar(DPT_FULL));
      };
      if (ok && niter > 0) {
        ok = issue_st(0);
        if (ok) issue_dpt(0);
      }
      for (int i = 0; i < niter && ok; ++i) {
        // P^T(i) is in S^T's columns: dV += P^T GH (query columns [0, 64)
        // of the A operand in TMEM columns [0, 32), [64, 128) in [64, 96)),
        // then S^T(i + 1) over them (in order).
        ok = mbar_wait(bar(PT_FULL), i & 1, abort_flag, 23);
        if (!ok) break;
        tc_fence_after();
        mma8_ts_mn_split(tmem + kColDV, tmem + kColS, sdesc(ga_of(i), 16384, 1024), id_mn,
                         i > 0 ? 1u : 0u);
        if (i + 1 < niter && !(ok = issue_st(i + 1))) break;
        // dS^T(i) is in dP^T's columns: dK += dS^T Q, then dP^T(i + 1).
        ok = mbar_wait(bar(DS_FULL), i & 1, abort_flag, 29);
        if (!ok) break;
        tc_fence_after();
        mma8_ts_mn_split(tmem + kColDK, tmem + kColDP, sdesc(qa_of(i), 16384, 1024), id_mn,
                         i > 0 ? 1u : 0u);
        mma_commit(bar(QG_EMPTY + (i & 1)));
        if (i + 1 < niter) issue_dpt(i + 1);
      }
      if (ok) mma_commit(bar(KV_DONE));
    }
    __syncwarp();
  } else {
    // ================================================= convert + epilogue
    const int hf = warp >> 2;
    const int kr = tid & 127;               // key row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    auto wait_all = [&](uint32_t b, uint32_t parity, uint32_t code) {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, code));
    };
    constexpr float kLog2e = 1.4426950408889634f;
    const float sl2 = A.scale * kLog2e;
    const int key = j0 + kr;
    // Per-query values of pair i in stage i & 1: four arrays of 128 (m =
    // c log2(e), r, Dc, j*), so four consecutive columns cost one broadcast
    // 16-byte shared load per array.  Thread t fills two of them for query
    // t & 127 (m and r, or Dc and j*).
    float* vec = reinterpret_cast<float*>(sbase + kVecOff);  // [stage][4][128]
    auto load_vec = [&](const QWalk& w, int i) {
      const int qi = tid & 127, which = tid >> 7;
      const int q = w.q0() + qi;
      const bool in = qi < w.qvalid();
      float* v = vec + (i & 1) * 512 + qi;
      const long long g = base_row + q;
      if (which == 0) {
        v[0] = in ? __ldg(A.c + g) * kLog2e : 0.f;
        v[128] = in ? __ldg(A.r + g) : 0.f;
      } else {
        v[256] = in ? __ldg(A.Dc + g) : 0.f;
        v[384] = __int_as_float(in ? __ldg(A.jstar + g) : -1);
      }
      mbar_arrive(bar(VEC_FULL + (i & 1)));
    };
    QWalk w{A.T, A.HW, A.Tc, A.To, A.nchunks, j0, j1};
    bool ok = w.seek(0);
    if (ok) load_vec(w, 0);
    for (int i = 0; i < niter && ok; ++i) {
      const int wk0 = w.w * A.HW, wk1 = w.end * A.HW;
      const bool key_in = key < j1 && key >= wk0 && key < wk1;
      const int qv = w.qvalid();
      ok = wait_all(bar(ST_FULL), i & 1, 24) && wait_all(bar(VEC_FULL + (i & 1)), (i >> 1) & 1, 25);
      if (!ok) break;
      tc_fence_after();
      const float4* vm = reinterpret_cast<const float4*>(vec + (i & 1) * 512);
      const float4* vr = vm + 32;
      const float4* vd = vm + 64;
      const float4* vj = vm + 96;
      // Every column of every row of the warp counts (the common case): no
      // per-element masks.
      const bool all_in = __all_sync(0xffffffffu, key_in) && qv == 128;
      // Phase 1: P^T = exp2(s scale log2(e) - m) of this half's 64 query
      // columns, written over them as bf16 pairs; kept in fp32 for phase 2.
      float pv[64];
      {
        uint32_t pp[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t xs[32];
          REHYAT_TMEM_LD32(lane_base + kColS + 64 * hf + 32 * c, xs);
          tmem_wait_ld();
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const int qa = 64 * hf + 32 * c + 4 * i4;
            const float4 m4 = vm[qa >> 2];
            const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i2 = 4 * i4 + e;
              const float p = ex2(fmaf(__uint_as_float(xs[i2]), sl2, -mm[e]));
              pv[32 * c + i2] = (all_in || (key_in && qa + e < qv)) ? p : 0.f;
            }
          }
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2) pp[16 * c + i2] = pack_bf16(pv[32 * c + 2 * i2], pv[32 * c + 2 * i2 + 1]);
        }
        REHYAT_TMEM_ST32(lane_base + kColS + 64 * hf, pp);
      }
      tmem_wait_st();
      // Q and GH rows past the chunk are zeroed before dV and dK read them
      // (their P and dS are 0; this keeps 0 * garbage out), once dP^T,
      // which reads GH, is done.
      if (qv < 128) ok = wait_all(bar(DPT_FULL), i & 1, 30);
      if (!ok) break;
      if (qv < 128 && kr >= qv) {
        const uint32_t qrow = base + kQOff + (i & 1) * 32768 + hf * 16384 + kr * 128;
        const uint32_t grow2 = base + kGOff + (i & 1) * 32768 + hf * 16384 + kr * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          st_shared_v4(qrow + c * 16, 0, 0, 0, 0);
          st_shared_v4(grow2 + c * 16, 0, 0, 0, 0);
        }
      }
      if (qv < 128) fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(PT_FULL));
      // Phase 2: dS^T = P^T (dP^T - r) - [j = j*] Dc over dP^T's columns.
      ok = wait_all(bar(DPT_FULL), i & 1, 30);
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t pd[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t xd[32];
          REHYAT_TMEM_LD32(lane_base + kColDP + 64 * hf + 32 * c, xd);
          tmem_wait_ld();
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const int qa = 64 * hf + 32 * c + 4 * i4;
            const float4 r4 = vr[qa >> 2];
            const int4 j4 = *reinterpret_cast<const int4*>(vj + (qa >> 2));
            const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
            const int jj[4] = {j4.x, j4.y, j4.z, j4.w};
            float d[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i2 = 4 * i4 + e;
              d[e] = pv[32 * c + i2] * (__uint_as_float(xd[i2]) - rr[e]);
            }
            // The maximum's term: this key is the arg-max of one of the
            // four queries (rare; masked queries carry j* = -1).
            if (jj[0] == key || jj[1] == key || jj[2] == key || jj[3] == key) {
              const float4 dc4 = vd[qa >> 2];
              const float dc[4] = {dc4.x, dc4.y, dc4.z, dc4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (jj[e] == key && key_in && qa + e < qv) d[e] -= dc[e];
            }
            pd[16 * c + 2 * i4] = pack_bf16(d[0], d[1]);
            pd[16 * c + 2 * i4 + 1] = pack_bf16(d[2], d[3]);
          }
        }
        REHYAT_TMEM_ST32(lane_base + kColDP + 64 * hf, pd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(DS_FULL));
      // The next pair's per-query values (stage (i + 1) & 1: every thread is
      // past pair i - 1, which used it).
      if (i + 1 < niter) {
        w.next();
        load_vec(w, i + 1);
      }
    }
    if (ok) ok = wait_all(bar(KV_DONE), 0, 26);
    if (ok) {
      tc_fence_after();
      // dv = dV, dk = scale dK; half hf writes columns [64 hf, 64 hf + 64).
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t ov[32], ok2[32];
        REHYAT_TMEM_LD32(lane_base + kColDV + 64 * hf + 32 * c, ov);
        REHYAT_TMEM_LD32(lane_base + kColDK + 64 * hf + 32 * c, ok2);
        tmem_wait_ld();
        if (key < j1) {
          float* dv = A.dv + (base_row + key) * 128 + 64 * hf + 32 * c;
          float* dk = A.dk + (base_row + key) * 128 + 64 * hf + 32 * c;
#pragma unroll
          for (int i2 = 0; i2 < 32; i2 += 4) {
            float4 v4 = make_float4(__uint_as_float(ov[i2]), __uint_as_float(ov[i2 + 1]),
                                    __uint_as_float(ov[i2 + 2]), __uint_as_float(ov[i2 + 3]));
            float4 k4 = make_float4(
                A.scale * __uint_as_float(ok2[i2]), A.scale * __uint_as_float(ok2[i2 + 1]),
                A.scale * __uint_as_float(ok2[i2 + 2]), A.scale * __uint_as_float(ok2[i2 + 3]));
            if (A.accumulate) {  // dk, dv already hold the linear branch's parts
              const float4 pv = *reinterpret_cast<const float4*>(dv + i2);
              const float4 pk = *reinterpret_cast<const float4*>(dk + i2);
              v4.x += pv.x; v4.y += pv.y; v4.z += pv.z; v4.w += pv.w;
              k4.x += pk.x; k4.y += pk.y; k4.z += pk.z; k4.w += pk.w;
            }
            *reinterpret_cast<float4*>(dv + i2) = v4;
            *reinterpret_cast<float4*>(dk + i2) = k4;
          }
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

}  // namespace

bool tc_attn_bwd_eligible(int in_bf16, int D) { return in_bf16 && D == 128 && encode_fn() != nullptr; }

cudaError_t launch_attn_bwd_dq_tc(const AttnBwdTcArgs& a, cudaStream_t s) {
  AttnBwdMaps maps;
  memset(&maps, 0, sizeof(maps));
  const long long N = static_cast<long long>(a.T) * a.HW;
  if (!make_map(&maps.q, a.q, N, a.BH) || !make_map(&maps.k, a.k, N, a.BH) ||
      !make_map(&maps.v, a.v, N, a.BH) || !make_map(&maps.gh, a.gh, N, a.BH))
    return cudaErrorInvalidValue;
  const cudaError_t e = ensure_smem(tc_bwd_dq_kernel, 8, bq::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int qrows_max = (a.Tc < a.T ? a.Tc : a.T) * a.HW;
  dim3 grid((qrows_max + 127) / 128, a.nchunks, a.BH);
  tc_bwd_dq_kernel<<<grid, bq::kThreads, bq::kSmemBytes, s>>>(maps, a);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_dkv_tc(const AttnBwdTcArgs& a, cudaStream_t s) {
  AttnBwdMaps maps;
  memset(&maps, 0, sizeof(maps));
  const long long N = static_cast<long long>(a.T) * a.HW;
  if (!make_map(&maps.q, a.q, N, a.BH) || !make_map(&maps.k, a.k, N, a.BH) ||
      !make_map(&maps.v, a.v, N, a.BH) || !make_map(&maps.gh, a.gh, N, a.BH))
    return cudaErrorInvalidValue;
  const cudaError_t e = ensure_smem(tc_bwd_dkv_kernel, 9, bk::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((N + 127) / 128), a.BH);
  tc_bwd_dkv_kernel<<<grid, bk::kThreads, bk::kSmemBytes, s>>>(maps, a);
  return cudaGetLastError();
}

}  // namespace rehyat
