// gsq_gemm_pair.cu -- the GSQ GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// C[M x N] = A[M x Kc] . B[N x Kc]^T, bf16 K-major operands, fp32 TMEM
// accumulators, epilogues as in the single-CTA kernel (gsq_gemm_epi.cuh).
//
// A cluster of two CTAs on neighbouring SMs owns a 256 x 256 output tile:
// CTA r loads rows [128 r, 128 r + 128) of the A tile and rows
// [128 r, 128 r + 128) of the B tile (half of the tile's N) into its own
// shared memory, in 64-wide K slabs through a 5-deep ring (32 KB per
// stage).  One thread of the leader CTA (rank 0) issues
// tcgen05.mma.cta_group::2 with M = 256, N = 256, which reads A and B from
// both CTAs and accumulates 128 rows into each CTA's TMEM.  Compared with a
// single CTA computing 128 x 256, each CTA moves a third fewer operand bytes
// per MMA, and the deeper ring hides more load latency.
//
// The epilogue stages each 32 x 32 piece of output in shared memory in the
// TMA swizzle layout and writes it with one TMA store (full lines, issued
// asynchronously), and reads Y_ref through TMA loads issued two pieces
// ahead; per-thread row-wise global accesses slowed the main loop.
//
// Both CTAs' TMA loads count their bytes on the leader's "full" barrier; the
// MMA thread signals each CTA's "empty" and "accumulator full" barriers with
// one tcgen05.commit per CTA (shared::cluster addresses from mapa); the
// epilogue warps of both CTAs release an accumulator on the leader's
// barrier.  Every TMA load lands in the issuing CTA's own shared memory
// only, from this GPU's own memory.  Every mbarrier wait
// is bounded; on timeout the kernel records DEV_ERR_TIMEOUT, drains what it
// issued, frees TMEM and returns.
#include "gsq_gemm_epi.cuh"

namespace gsq {

namespace {

constexpr int PM = 256, HALF = 128, BK = 64;
constexpr int A_BYTES = HALF * BK * 2;
constexpr int NUM_THREADS = 192;
constexpr long long WAIT_LIMIT = 4000000000LL;  // clock cycles (~2 s)
constexpr long long PROBE_LIMIT = 20000000LL;   // the test hook's wait (~10 ms)

// Output tile width BN (256, or 128 for N = 128 problems): each CTA loads
// BN / 2 rows of B per stage; two BN-column TMEM accumulators per CTA.
template <int BN>
struct Cfg {
  static constexpr int PN = BN;
  static constexpr int HALFN = BN / 2;
  static constexpr int STAGES = BN == 256 ? 5 : 6;
  static constexpr int B_BYTES = HALFN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr uint32_t IDESC = idesc_bf16_f32(PM, BN);
  static constexpr int UNITS = BN / 32;
};

template <int STAGES>
struct Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t done;
  uint64_t ybar[4][2];  // Y_ref tile loads of each epilogue warp
  uint64_t probe;       // test hook: a barrier nothing arrives at
  uint32_t tmem_base;
  int abort;
  double red[4];
};

// Epilogue staging per epilogue warp (32 rows x 32 columns per unit, two
// buffers each): fp32 out tiles 4 KB, Y_ref tiles 4 KB, bf16 dY tiles 2 KB.
constexpr int OUT_TILE = 32 * 32 * 4;
constexpr int DY_TILE = 32 * 32 * 2;
template <int EPI>
__host__ __device__ constexpr int warp_stage_bytes() {
  return EPI == EPI_STORE_BF16 ? 2 * DY_TILE
                               : ((EPI == EPI_LOSS_DY || EPI == EPI_MERGED)
                                      ? 2 * OUT_TILE + 2 * DY_TILE
                                      : 2 * OUT_TILE);
}
template <int EPI, int BN>
__host__ __device__ constexpr int smem_bytes() {
  return Cfg<BN>::STAGES * Cfg<BN>::STAGE_BYTES + 4 * warp_stage_bytes<EPI>() + 1024 +
         (int)sizeof(Ctl<Cfg<BN>::STAGES>);
}

// Where tile `tile` of a launch sits: problem offsets, tile origin, and its
// K range (see GemmSched).
struct TileAt {
  int64_t a_row, a_k, b_row, b_k, o_row, o_col;  // origin of the problem
  int64_t m0, n0;  // tile origin inside the problem
  int64_t r0;      // causal: tile rows' position inside their period
  int nk;          // K blocks of 64
  int kps;         // causal = 2: K blocks per period
};

template <int BN>
__device__ __forceinline__ TileAt tile_at(int tile, int m_tiles, int n_tiles,
                                          int64_t Kc, const GemmSched& sc) {
  TileAt t;
  int mb, nb, p;
  t.r0 = 0;
  t.kps = 0;
  if (sc.causal == 0) {
    const int per = m_tiles * n_tiles;
    p = tile / per;
    const int local = tile - p * per;
    if (sc.group_m > 1) {
      // bands of group_m row tiles: a wave of CTA pairs then shares a few
      // row tiles of A and a few column tiles of B instead of streaming one
      // row tile of A per pair
      const int band_tiles = sc.group_m * n_tiles;
      const int band = local / band_tiles;
      const int within = local - band * band_tiles;
      const int first = band * sc.group_m;
      const int gm = m_tiles - first < sc.group_m ? m_tiles - first : sc.group_m;
      mb = first + within % gm;
      nb = within / gm;
    } else {
      mb = local % m_tiles;
      nb = local / m_tiles;
    }
    t.nk = (int)((Kc + BK - 1) / BK);
    if (sc.nseg > 1) t.kps = (int)(sc.seg / BK);
  } else {
    // the period position is the slowest index, longest K first
    const int rbs = (int)(sc.seg / PM);
    const int hs = m_tiles / rbs;
    const int per = sc.count * n_tiles * hs;
    const int j = tile / per;
    int rest = tile - j * per;
    const int hseg = rest % hs;
    rest /= hs;
    nb = rest % n_tiles;
    p = rest / n_tiles;
    const int rb = sc.causal == 1 ? rbs - 1 - j : j;
    mb = hseg * rbs + rb;
    t.r0 = (int64_t)rb * PM;
    if (sc.causal == 1) {
      const int64_t kend = t.r0 + PM < Kc ? t.r0 + PM : Kc;
      t.nk = (int)((kend + BK - 1) / BK);
    } else {
      t.kps = (int)((sc.seg - t.r0) / BK);
      t.nk = sc.nseg * t.kps;
    }
  }
  const int64_t p1 = p / sc.inner, p2 = p - p1 * sc.inner;
  t.a_row = sc.a_row[0] * p1 + sc.a_row[1] * p2;
  t.a_k = sc.a_k[0] * p1 + sc.a_k[1] * p2;
  t.b_row = sc.b_row[0] * p1 + sc.b_row[1] * p2;
  t.b_k = sc.b_k[0] * p1 + sc.b_k[1] * p2;
  t.o_row = sc.o_row[0] * p1 + sc.o_row[1] * p2;
  t.o_col = sc.o_col[0] * p1 + sc.o_col[1] * p2;
  t.m0 = (int64_t)mb * PM;
  t.n0 = (int64_t)nb * BN;
  return t;
}

// TMA coordinates of K block kb of a tile: A and B column (K) and the row
// offset each operand adds for its K segment
struct KAt {
  int64_t ak, bk, arow, brow;
};
__device__ __forceinline__ KAt tile_k(const TileAt& t, int kb, const GemmSched& sc) {
  KAt k;
  if (sc.causal != 2 && sc.nseg <= 1) {
    k.ak = t.a_k + (int64_t)kb * BK;
    k.bk = t.b_k + (int64_t)kb * BK;
    k.arow = k.brow = 0;
    return k;
  }
  const int sgi = kb / t.kps;
  const int64_t within = t.r0 + (int64_t)(kb - sgi * t.kps) * BK;
  k.ak = t.a_k + sgi * sc.a_seg_k + within;
  k.bk = t.b_k + sgi * sc.b_seg_k + within;
  k.arow = sgi * sc.a_seg_row;
  k.brow = sgi * sc.b_seg_row;
  return k;
}

// shared-memory offset of 16-byte chunk j of row r in a tile written or
// read by TMA with 128-byte rows / 128-byte swizzle, or 64-byte rows /
// 64-byte swizzle (the tile base is 1024-byte aligned)
__device__ __forceinline__ uint32_t swz128(int r, int j) {
  return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint32_t swz64(int r, int j) {
  return (uint32_t)(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

// acquire load of a counter another CTA releases; then the fence that orders
// it before this thread's later async-proxy (TMA) reads of global memory
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Row band of a merged launch's tile and whether it is a weight-gradient
// tile: forward tiles [0, tiles_f) first, then the weight-gradient tiles,
// each problem with its column tiles fastest inside a band of 256 rows.
__device__ __forceinline__ TileAt merged_tile_at(int tile, int tiles_f, int n_tiles,
                                                 int n_tiles2, int64_t Kc, int64_t Kc2,
                                                 bool& wgrad) {
  TileAt t;
  wgrad = tile >= tiles_f;
  const int local = wgrad ? tile - tiles_f : tile;
  const int nt = wgrad ? n_tiles2 : n_tiles;
  t.a_row = t.a_k = t.b_row = t.b_k = t.o_row = t.o_col = 0;
  t.r0 = 0;
  t.kps = 0;
  t.m0 = (int64_t)(local / nt) * PM;
  t.n0 = (int64_t)(local % nt) * 256;
  t.nk = (int)(((wgrad ? Kc2 : Kc) + BK - 1) / BK);
  return t;
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  const bool ok = mbar_wait_bounded(bar, parity, WAIT_LIMIT);
  return __all_sync(0xffffffffu, ok);
}

template <int EPI, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA,
                const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmO,
                const __grid_constant__ CUtensorMap tmY, int64_t M, int64_t N,
                int64_t Kc, EpiParams ep, const __grid_constant__ GemmSched sc,
                const __grid_constant__ MergeArgs mg) {
  pdl_trigger();  // our CTAs are all resident (persistent grid)
  using C = Cfg<BN>;
  // a merged launch: forward tiles (loss + dY epilogue) then weight-gradient
  // tiles (fp32 store into mg.tmO2)
  constexpr bool MERGED = EPI == EPI_MERGED;
  constexpr int PN = C::PN, STAGES = C::STAGES, STAGE_BYTES = C::STAGE_BYTES;
  constexpr int TMEM_COLS = C::TMEM_COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_area = smem + STAGES * STAGE_BYTES;
  auto* ctl = reinterpret_cast<Ctl<STAGES>*>(stage_area + 4 * warp_stage_bytes<EPI>());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int m_tiles = (int)((M + PM - 1) / PM);
  const int n_tiles = (int)((N + PN - 1) / PN);
  const int n_tiles2 = MERGED ? (int)((mg.N2 + PN - 1) / PN) : 0;
  const int tiles_f = m_tiles * n_tiles * sc.count;
  // the test hook's launch processes no tile: nothing is ever in flight
  const int num_tiles = ep.stall_probe ? 0 : tiles_f + (MERGED ? m_tiles * n_tiles2 : 0);
  // where tile `tile` sits, and whether it is a merged launch's weight-gradient tile
  auto at = [&](int tile, bool& wgrad) -> TileAt {
    if (MERGED) return merged_tile_at(tile, tiles_f, n_tiles, n_tiles2, Kc, mg.Kc2, wgrad);
    wgrad = false;
    return tile_at<BN>(tile, m_tiles, n_tiles, Kc, sc);
  };
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctl->tfull[b]), 1);
      mbar_init(smem_u32(&ctl->tempty[b]), 8);  // 4 epilogue warps x 2 CTAs
    }
    mbar_init(smem_u32(&ctl->done), 1);
    for (int w = 0; w < 4; ++w)
      for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&ctl->ybar[w][b]), 1);
    mbar_init(smem_u32(&ctl->probe), 1);
    ctl->abort = 0;
    mbar_fence_init();
    if (EPI != EPI_LOSS) tma_prefetch_desc(&tmO);
    if (EPI == EPI_LOSS_DY || EPI == EPI_LOSS || MERGED || EPI == EPI_SUB_F32)
      tma_prefetch_desc(&tmY);
    if (MERGED) {
      tma_prefetch_desc(&mg.tmA2);
      tma_prefetch_desc(&mg.tmB2);
      tma_prefetch_desc(&mg.tmO2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote access
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  // the setup above overlapped the previous kernel's tail; its outputs (our
  // operands) and its reads of what we write are complete after this
  pdl_wait();
  if (ep.stall_probe && threadIdx.x == 0) {
    // a bounded wait that runs out: the error word reports it
    if (!mbar_wait_bounded(smem_u32(&ctl->probe), 0, PROBE_LIMIT))
      atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
  }

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        bool wgrad;
        const TileAt ta = at(tile, wgrad);
        const int32_t ya = (int32_t)(ta.a_row + ta.m0 + (int)rank * HALF);
        const int32_t yb = (int32_t)(ta.b_row + ta.n0 + (int)rank * C::HALFN);
        const void* mapA = &tmA;
        const void* mapB = &tmB;
        if (MERGED && wgrad) {
          mapA = &mg.tmA2;
          mapB = &mg.tmB2;
          // this band's dY rows must be in memory: every forward tile of the
          // band has counted its stores (bounded wait)
          const unsigned* flag = mg.band_done + ta.m0 / PM;
          if (ld_acquire_u32(flag) < mg.target) {
            const long long t0 = clock64();
            while (ld_acquire_u32(flag) < mg.target) {
              if (clock64() - t0 > WAIT_LIMIT || *(volatile int*)&ctl->abort) {
                ok = false;
                break;
              }
              __nanosleep(128);
            }
            if (!ok) break;
          }
          fence_proxy_async_global();
        }
        for (int kb = 0; kb < ta.nk; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&ctl->empty[stage]), ph ^ 1,
                                 WAIT_LIMIT) ||
              *(volatile int*)&ctl->abort) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&ctl->full[stage]);
          const uint32_t fb_leader = mapa_shared(fb, 0);
          if (leader) mbar_arrive_expect_tx(fb, 2 * STAGE_BYTES);
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          const KAt kx = tile_k(ta, kb, sc);
          tma_load_2d_pair(sa, mapA, fb_leader, (int32_t)kx.ak, ya + (int32_t)kx.arow);
          tma_load_2d_pair(sa + A_BYTES, mapB, fb_leader, (int32_t)kx.bk,
                           yb + (int32_t)kx.brow);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
        *(volatile int*)&ctl->abort = 1;
      }
      // drain (leader): the last phase armed on each stage has completed,
      // i.e. both CTAs' loads into it have landed
      if (leader) {
        for (int s = 0; s < STAGES; ++s) {
          if (issued <= s) break;
          const long long last = ((issued - 1 - s) / STAGES) * STAGES + s;
          const uint32_t par = (uint32_t)((last / STAGES) & 1);
          if (!mbar_wait_bounded(smem_u32(&ctl->full[s]), par, WAIT_LIMIT))
            atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // --------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        if (!mbar_wait_bounded(smem_u32(&ctl->tempty[acc]), aph ^ 1,
                               WAIT_LIMIT)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * PN);
        bool wgrad_unused;
        const int nk = at(tile, wgrad_unused).nk;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), ph,
                                 WAIT_LIMIT) ||
              *(volatile int*)&ctl->abort) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          const uint64_t ad = sdesc_kmajor_sw128(sa);
          const uint64_t bd = sdesc_kmajor_sw128(sa + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16_pair(d_tmem, ad + 2 * k, bd + 2 * k, C::IDESC,
                           (kb > 0 || k > 0) ? 1u : 0u);
          const uint32_t eb = smem_u32(&ctl->empty[stage]);
          umma_commit_pair(mapa_shared(eb, 0));
          umma_commit_pair(mapa_shared(eb, 1));
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        const uint32_t tb = smem_u32(&ctl->tfull[acc]);
        umma_commit_pair(mapa_shared(tb, 0));
        umma_commit_pair(mapa_shared(tb, 1));
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      if (!ok) {
        atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
        *(volatile int*)&ctl->abort = 1;
      }
      // drain: every MMA this thread issued has completed
      umma_commit_pair(mapa_shared(smem_u32(&ctl->done), 0));
      if (!mbar_wait_bounded(smem_u32(&ctl->done), 0, WAIT_LIMIT))
        atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------- epilogue
    // Warp w (2..5) drains TMEM lanes [32 q, 32 q + 32), q = w % 4, in units
    // of 32 columns: tcgen05.ld -> registers -> (Y_ref from a TMA-loaded
    // tile) -> swizzled shared-memory tile -> one TMA store of 32 x 32.
    const int q = warp & 3;
    const int ew = warp - 2;
    uint8_t* wst = stage_area + ew * warp_stage_bytes<EPI>();
    const uint32_t out_s = smem_u32(wst);                  // 2 x OUT_TILE
    const uint32_t y_s = smem_u32(wst);                    // 2 x OUT_TILE
    const uint32_t dy_s = smem_u32(wst + 2 * OUT_TILE);    // 2 x DY_TILE
    constexpr int UNITS = C::UNITS;
    const int my_tiles = pair < num_tiles ? (num_tiles - 1 - pair) / npairs + 1 : 0;
    // units that read Y_ref: all of them, or a merged launch's forward ones
    // (a pair's forward tiles come before its weight-gradient tiles)
    const int fwd_tiles_mine =
        MERGED ? (pair < tiles_f ? (tiles_f - 1 - pair) / npairs + 1 : 0) : my_tiles;
    const int64_t y_units = (int64_t)(fwd_tiles_mine < my_tiles ? fwd_tiles_mine : my_tiles) * UNITS;
    // coordinates (x = column, y = first row) of unit u of this warp; false
    // when the unit lies wholly outside its problem's M x N
    auto unit_xy = [&](int64_t u, int32_t& x, int32_t& y) {
      const int tile = pair + (int)(u / UNITS) * npairs;
      bool wgrad;
      const TileAt ta = at(tile, wgrad);
      const int64_t ncols = (MERGED && wgrad) ? mg.N2 : N;
      const int64_t lx = ta.n0 + (int)(u % UNITS) * 32;
      const int64_t ly = ta.m0 + (int)rank * HALF + q * 32;
      if (sc.o_fold > 0) {
        const int64_t f = ly / sc.o_fold;
        x = (int32_t)(ta.o_col + f * sc.o_fold_col + lx);
        y = (int32_t)(ta.o_row + (ly - f * sc.o_fold));
      } else {
        x = (int32_t)(ta.o_col + lx);
        y = (int32_t)(ta.o_row + ly);
      }
      return lx < ncols && ly < M;
    };
    int64_t y_issued = 0;
    auto issue_y = [&](int64_t u) {  // lane 0: Y_ref tile of unit u
      int32_t x, y;
      unit_xy(u, x, y);
      const uint32_t bar = smem_u32(&ctl->ybar[ew][u & 1]);
      mbar_arrive_expect_tx(bar, OUT_TILE);
      tma_load_2d(y_s + (uint32_t)((u & 1) * OUT_TILE), &tmY, bar, x, y);
    };
    if ((EPI == EPI_LOSS_DY || EPI == EPI_LOSS || MERGED || EPI == EPI_SUB_F32) && lane == 0) {
      for (; y_issued < 2 && y_issued < y_units; ++y_issued) issue_y(y_issued);
    }
    int acc = 0;
    uint32_t aph = 0;
    double lsum = 0.0;
    int64_t u = 0;
    int last_buf = -1;  // staging buffer of the newest committed store (lane 0)
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
      // a merged launch's weight-gradient tile takes the fp32-store epilogue,
      // its forward tiles the loss + dY one
      bool wtile = false;
      int64_t band = 0;
      if (MERGED) band = at(tile, wtile).m0 / PM;
      const bool store_f32 = EPI == EPI_STORE_F32 || (MERGED && wtile);
      const bool store_any = store_f32 || EPI == EPI_STORE_BF16;
      const bool with_dy = EPI == EPI_LOSS_DY || (MERGED && !wtile);
      const void* mapO = (MERGED && wtile) ? (const void*)&mg.tmO2 : (const void*)&tmO;
      if (!warp_wait(smem_u32(&ctl->tfull[acc]), aph) ||
          *(volatile int*)&ctl->abort) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * PN);
      float part = 0.f;
#pragma unroll 1
      for (int c = 0; c < UNITS; ++c, ++u) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), v);
        tmem_wait_ld();
        int32_t x, y;
        const bool inside = unit_xy(u, x, y);
        const int b = (int)(u & 1);
        if (store_any) {
          // this buffer may be rewritten once the store that last read it is
          // done: the newest group if it used this buffer, else the one before
          if (lane == 0) {
            if (last_buf == b) bulk_wait_read<0>();
            else bulk_wait_read<1>();
          }
          __syncwarp();
          const uint32_t base = out_s + (uint32_t)(b * (store_f32 ? OUT_TILE : DY_TILE));
          if (store_f32) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint32_t a = base + swz128(lane, j);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                           "r"(v[4 * j]), "r"(v[4 * j + 1]), "r"(v[4 * j + 2]),
                           "r"(v[4 * j + 3])
                           : "memory");
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t a = base + swz64(lane, j);
              const float* f = reinterpret_cast<const float*>(v) + 8 * j;
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                           "r"(pack_bf16x2(f[0], f[1])), "r"(pack_bf16x2(f[2], f[3])),
                           "r"(pack_bf16x2(f[4], f[5])), "r"(pack_bf16x2(f[6], f[7]))
                           : "memory");
            }
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0 && inside) {  // no store for a box wholly outside C
            tma_store_2d(mapO, base, x, y);
            bulk_commit();
            last_buf = b;
          }
        } else {
          // Y_ref of this unit, loaded by TMA (zero outside the matrix)
          if (!warp_wait(smem_u32(&ctl->ybar[ew][b]), (uint32_t)((u >> 1) & 1))) {
            ok = false;
            break;
          }
          const uint32_t ybase = y_s + (uint32_t)(b * OUT_TILE);
          float e[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 y4;
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(y4.x), "=f"(y4.y), "=f"(y4.z), "=f"(y4.w)
                         : "r"(ybase + swz128(lane, j))
                         : "memory");
            e[4 * j] = __uint_as_float(v[4 * j]) - y4.x;
            e[4 * j + 1] = __uint_as_float(v[4 * j + 1]) - y4.y;
            e[4 * j + 2] = __uint_as_float(v[4 * j + 2]) - y4.z;
            e[4 * j + 3] = __uint_as_float(v[4 * j + 3]) - y4.w;
          }
          if (EPI == EPI_SUB_F32) {
            // C - acc = -e goes back into the slots this lane just read,
            // and out by TMA; the buffer is loaded again only after the
            // store has read it
#pragma unroll
            for (int j = 0; j < 8; ++j)
              asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                               ybase + swz128(lane, j)),
                           "f"(-e[4 * j]), "f"(-e[4 * j + 1]), "f"(-e[4 * j + 2]),
                           "f"(-e[4 * j + 3])
                           : "memory");
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (inside) {
                tma_store_2d(&tmO, ybase, x, y);
                bulk_commit();
              }
              bulk_wait_read<0>();
            }
          }
          __syncwarp();  // every lane has read this Y_ref buffer
          if (lane == 0 && y_issued < y_units && y_issued == u + 2) {
            issue_y(y_issued);
            ++y_issued;
          }
          if (EPI != EPI_SUB_F32) {
#pragma unroll
            for (int j = 0; j < 32; ++j) part = fmaf(e[j], e[j], part);
          }
          if (with_dy) {
            if (lane == 0) {
              if (last_buf == b) bulk_wait_read<0>();
              else bulk_wait_read<1>();
            }
            __syncwarp();
            const uint32_t dbase = dy_s + (uint32_t)(b * DY_TILE);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t a = dbase + swz64(lane, j);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                           "r"(pack_bf16x2(2.f * e[8 * j], 2.f * e[8 * j + 1])),
                           "r"(pack_bf16x2(2.f * e[8 * j + 2], 2.f * e[8 * j + 3])),
                           "r"(pack_bf16x2(2.f * e[8 * j + 4], 2.f * e[8 * j + 5])),
                           "r"(pack_bf16x2(2.f * e[8 * j + 6], 2.f * e[8 * j + 7]))
                           : "memory");
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0 && inside) {
              tma_store_2d(mapO, dbase, x, y);
              bulk_commit();
              last_buf = b;
            }
          }
        }
      }
      lsum += (double)part;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&ctl->tempty[acc]), 0));
      if (MERGED && !wtile && ok && lane == 0) {
        // this warp's dY stores of the tile are complete: count them for the
        // band's weight-gradient tiles (the async-proxy writes are ordered
        // before the release of the count)
        bulk_wait_all();
        fence_proxy_async_global();
        __threadfence();
        atomicAdd(mg.band_done + band, 1u);
      }
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
    if (!ok && lane == 0) {
      atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
      *(volatile int*)&ctl->abort = 1;
    }
    if (lane == 0) {
      // Y_ref loads still in flight land before the CTA exits
      for (int64_t k = u; k < y_issued; ++k)
        if (!mbar_wait_bounded(smem_u32(&ctl->ybar[ew][k & 1]),
                               (uint32_t)((k >> 1) & 1), WAIT_LIMIT))
          atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
      bulk_wait_all();  // stores complete before the CTA exits
    }
    __syncwarp();
    if (EPI == EPI_LOSS_DY || EPI == EPI_LOSS || MERGED) {
      lsum = warp_sum_d(lsum);
      if (lane == 0) ctl->red[q] = lsum;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (warp == 2 && lane == 0)
        loss_finish(ctl->red[0] + ctl->red[1] + ctl->red[2] + ctl->red[3], ep);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its pair may still touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// Band height of the tile order (GemmSched::group_m) when the caller leaves it
// to the launcher: bands of 8 row tiles once A has 24 or more row tiles (its
// row tiles then no longer stay in L2 from one column tile to the next; a
// wave of 74 pairs reads about 19 distinct operand tiles instead of about 75
// on the 70B MLP shapes), row tiles fastest otherwise.
inline int auto_group_m(int m_tiles, int n_tiles) {
  return (m_tiles >= 24 && n_tiles > 1) ? 8 : 1;
}

template <int EPI, int BN>
cudaError_t launch_pair_epi(const CUtensorMap& tmA, const CUtensorMap& tmB,
                            const EpiMaps& maps, int64_t M, int64_t N,
                            int64_t Kc, const GemmSched& sc_in, const EpiParams& ep,
                            int sm_count, cudaStream_t st,
                            const MergeArgs& mg = MergeArgs()) {
  GemmSched sc = sc_in;
  if (sc.causal == 0 && sc.group_m == 0)
    sc.group_m = auto_group_m((int)((M + PM - 1) / PM), (int)((N + BN - 1) / BN));
  // co-resident CTA pairs of this kernel (the same on every B200; computed once)
  static std::atomic<int> max_pairs_cache{0};
  int max_pairs = max_pairs_cache.load(std::memory_order_relaxed);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = smem_bytes<EPI, BN>();
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below takes the cluster shape only
  {
    const cudaError_t e = smem_optin<k_gemm_pair<EPI, BN>>(smem_bytes<EPI, BN>());
    if (e != cudaSuccess) return e;
  }
  if (max_pairs == 0) {
    cfg.gridDim = dim3((unsigned)(2 * (sm_count / 2)));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_gemm_pair<EPI, BN>, &cfg) != cudaSuccess ||
        n <= 0) {
      cudaGetLastError();
      n = sm_count / 2;
    }
    max_pairs = n;
    max_pairs_cache.store(n, std::memory_order_relaxed);
  }
  int64_t tiles = ((M + PM - 1) / PM) * ((N + BN - 1) / BN) * (int64_t)sc.count;
  if (EPI == EPI_MERGED) tiles = merged_tiles(M, N, mg.N2);
  const int pairs = (int)(tiles < max_pairs ? tiles : max_pairs);
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_gemm_pair<EPI, BN>, tmA, tmB, maps.out, maps.yref,
                            M, N, Kc, ep, sc, mg);
}

}  // namespace

cudaError_t launch_gemm_pair(const CUtensorMap& tmA, const CUtensorMap& tmB,
                             const EpiMaps& maps, int64_t M, int64_t N,
                             int64_t Kc, int mode, const EpiParams& ep,
                             int sm_count, cudaStream_t st) {
  const GemmSched one;
  switch (mode) {
    case EPI_STORE_F32:
      return launch_pair_epi<EPI_STORE_F32, 256>(tmA, tmB, maps, M, N, Kc, one, ep,
                                                 sm_count, st);
    case EPI_LOSS_DY:
      return launch_pair_epi<EPI_LOSS_DY, 256>(tmA, tmB, maps, M, N, Kc, one, ep,
                                               sm_count, st);
    case EPI_STORE_BF16:
      return launch_pair_epi<EPI_STORE_BF16, 256>(tmA, tmB, maps, M, N, Kc, one, ep,
                                                  sm_count, st);
    case EPI_SUB_F32:
      return launch_pair_epi<EPI_SUB_F32, 256>(tmA, tmB, maps, M, N, Kc, one, ep,
                                               sm_count, st);
    default:
      return launch_pair_epi<EPI_LOSS, 256>(tmA, tmB, maps, M, N, Kc, one, ep, sm_count,
                                            st);
  }
}

int64_t merged_band_tiles(int64_t N) { return (N + 255) / 256; }

int64_t merged_tiles(int64_t M, int64_t N, int64_t N2) {
  return ((M + PM - 1) / PM) * (merged_band_tiles(N) + merged_band_tiles(N2));
}

cudaError_t launch_gemm_merged(const CUtensorMap& tmA, const CUtensorMap& tmB,
                               const EpiMaps& maps, int64_t M, int64_t N, int64_t Kc,
                               const MergeArgs& mg, const EpiParams& ep, int sm_count,
                               cudaStream_t st) {
  if (M <= 0 || N <= 0 || Kc <= 0 || mg.N2 <= 0 || mg.Kc2 <= 0 || !mg.band_done)
    return cudaErrorInvalidValue;
  const GemmSched one;
  return launch_pair_epi<EPI_MERGED, 256>(tmA, tmB, maps, M, N, Kc, one, ep, sm_count, st,
                                           mg);
}

cudaError_t launch_gemm_batched(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const CUtensorMap& tmOut, int64_t M, int64_t N,
                                int64_t Kc, int bn, const GemmSched& sc, int mode,
                                const EpiParams& ep, int sm_count, cudaStream_t st) {
  if (sc.count < 1 || sc.inner < 1 || M <= 0 || N <= 0 || Kc <= 0 || Kc % BK)
    return cudaErrorInvalidValue;
  if (sc.causal < 0 || sc.causal > 2 || sc.nseg < 1) return cudaErrorInvalidValue;
  if (sc.nseg > 1 || sc.causal == 2) {
    if (sc.seg <= 0 || sc.seg % BK || Kc != sc.seg * sc.nseg) return cudaErrorInvalidValue;
    if (sc.causal == 1) return cudaErrorInvalidValue;
  }
  if (sc.causal) {
    if (sc.seg <= 0 || sc.seg % PM) return cudaErrorInvalidValue;
    if (sc.causal == 1 && M % sc.seg) return cudaErrorInvalidValue;
    if (sc.causal == 2 && M != sc.seg) return cudaErrorInvalidValue;
  }
  EpiMaps maps;
  maps.out = tmOut;
  maps.yref = tmOut;
  if (sc.o_fold < 0 || (sc.o_fold > 0 && sc.o_fold % 32)) return cudaErrorInvalidValue;
  if (mode == EPI_STORE_F32 && bn == 128)
    return launch_pair_epi<EPI_STORE_F32, 128>(tmA, tmB, maps, M, N, Kc, sc, ep, sm_count,
                                               st);
  if (mode == EPI_STORE_F32 && bn == 256)
    return launch_pair_epi<EPI_STORE_F32, 256>(tmA, tmB, maps, M, N, Kc, sc, ep, sm_count,
                                               st);
  if (mode == EPI_STORE_BF16 && bn == 128)
    return launch_pair_epi<EPI_STORE_BF16, 128>(tmA, tmB, maps, M, N, Kc, sc, ep, sm_count,
                                                st);
  if (mode == EPI_STORE_BF16 && bn == 256)
    return launch_pair_epi<EPI_STORE_BF16, 256>(tmA, tmB, maps, M, N, Kc, sc, ep, sm_count,
                                                st);
  return cudaErrorInvalidValue;
}

}  // namespace gsq
