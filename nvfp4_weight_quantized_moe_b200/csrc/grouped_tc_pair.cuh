// Pair form of the tcgen05 projection kernel, for experts with many token
// rows (prefill-shaped batches).  Part of grouped_tc.cu (included there once,
// after the one-CTA kernel): it uses that file's packing, tensor maps and
// arguments.
//
// A cluster of two CTAs runs tcgen05.mma.cta_group::2: M = 256 weight rows
// (128 per CTA, each decoded into its own CTA's tensor or shared memory) times
// N = up to NT token rows (256 or 192 for prefill-shaped batches, 32 for
// decode-shaped ones; each CTA loads half of the token tile into its own
// shared memory), FP32 accumulators in both CTAs' tensor memory (each CTA
// holds its 128 rows x all N columns).  Per FLOP this halves the decode work and the
// tensor-memory stores of the one-CTA kernel at 128-token passes and cuts its
// shared-memory traffic by a third, which is what bounded that kernel's MMA
// rate.
//
// Rows.  Gate+up: CTA r of the pair owns outputs n0 + 64 r .. + 63, and its
// 128 A rows interleave them: TMEM lane 2j holds gate row n0 + 64 r + j, lane
// 2j + 1 the up row of the same n, so the SiLU(gate) * up epilogue pairs
// neighbouring lanes with one shuffle.  Down and up+activation: CTA r owns 128
// consecutive rows n0 + 128 r .. + 127 of the one matrix.
//
// Roles (15 warps per CTA), synchronised by mbarriers only:
//   warps 0-7   decoders: A row 32 (w % 4) + l, the 64-k stages of parity
//               w / 4; 32 nibble bytes and 4 scales per stage from the weight
//               tile in shared memory, exact E2M1 x E4M3 -> f16, into the A
//               ring (tcgen05.st into tensor memory, or, at 256-row passes,
//               128-byte-swizzled rows in shared memory); each warp then
//               arrives on the first CTA's full_a barrier (the peer's warps
//               remotely);
//   warp 8      first CTA: MMA issuer (one thread): per two stages, waits
//               for their full_a barriers (both CTAs' A stage; one decoder
//               lane folds in the token tile's arrival), issues the pair MMAs
//               into one of two D buffers and commits once; each pass ends
//               with a commit too; commits reach barriers in both CTAs
//               (multicast commit);
//   warp 9      weight tiles by TMA (its CTA's 128 rows, 256 k per tile);
//   warp 10     token tiles by TMA, its half of each 64-k stage, completion
//               signalled on the first CTA's full_b barrier (pair TMA form);
//   warps 11-14 epilogue: tcgen05.ld of the finished D buffer, FP32 scaling,
//               SiLU(g) * u or the activation, stores by sorted position, then
//               the D buffer is handed back (remote arrive for the peer).
// D is double-buffered, so a pass's epilogue overlaps the next pass's MMAs.
// Every wait is bounded; on timeout the CTA flags the device error word and
// skips its remaining waits; both CTAs meet at a cluster barrier before the
// tensor memory is freed.

namespace {

constexpr int kPairMmaWarp = 8;
constexpr int kPairWLoadWarp = 9;
constexpr int kPairBLoadWarp = 10;
constexpr int kPairEpiWarp0 = 11;           // warps 11..14
constexpr int kPairThreads = 32 * 15;
constexpr int kPairWBoxRows = 64;           // rows per weight TMA box
constexpr int kPairWNib = 128 * 128;        // nibble bytes of a CTA's weight tile (128 rows x 256 k)
constexpr int kPairWSlot = kPairWNib + 128 * 16;

// NT: token rows per pass of the pair (the MMA's N at most): 256 for gate+up
// of experts with many rows, with the A operand in shared memory (two 256-column
// accumulators fill tensor memory); 192 for down of such experts (A in tensor
// memory; its hi + lo token planes leave no shared memory for A); 32 for
// decode-shaped batches (two pairs per SM pair, each with its own MMA issuer
// and weight stream; A in tensor memory).
template <int MODE, int NT>
struct PairCfg {
  static constexpr bool SMEM_A = NT == 256;                           // A operand in shared memory
  static constexpr int HALF = NT / 2;                                 // token rows each CTA loads
  static constexpr int CTAS_PER_SM = NT > 32 ? 1 : 2;
  static constexpr int PLANES = MODE == kModeDown ? 2 : 1;           // down: f16 hi + lo
  static constexpr int ROWS_PER_PAIR = MODE == kModeGateUp ? 128 : 256;  // outputs n per pair
  static constexpr int B_PLANE_BYTES = HALF * kStageK * 2;           // HALF rows x 64 k f16
  static constexpr int B_SLOT_BYTES = PLANES * B_PLANE_BYTES;
  static constexpr int A_COLS = 32;                                   // TMEM columns per A stage (A in TMEM)
  static constexpr int A_STAGE_BYTES = 128 * kStageK * 2;             // 128 rows x 64 k f16 (A in smem)
  static constexpr int D_COLS = NT;                                   // per D buffer
  static constexpr int ND = 2;                                        // D buffers
  static constexpr int WS = SMEM_A ? 2 : 3;
  static constexpr int SB = SMEM_A ? 6 : (MODE == kModeDown && NT > 32) ? 4 : 8;
  static constexpr uint32_t TMEM_COLS = 512 / CTAS_PER_SM;
  // A ring: the rest of the CTA's tensor memory, at most SB stages (the
  // completion ring of SB entries also tells the decoders when an A slot is free).
  static constexpr int SA_TMEM = ((int)TMEM_COLS - ND * D_COLS) / A_COLS;
  static constexpr int SA = SMEM_A ? 4 : (SA_TMEM < SB ? SA_TMEM : SB);
  static constexpr int OFF_W = 0;
  static constexpr int OFF_B = WS * kPairWSlot;
  static constexpr int OFF_A = OFF_B + SB * B_SLOT_BYTES;             // A ring (A in smem only)
  static constexpr int OFF_BAR = OFF_A + (SMEM_A ? SA * A_STAGE_BYTES : 0);
  // full_w[WS], empty_w[WS], full_b[SB], mma_done[SB], full_a[SA], done[ND], dfree[ND]
  static constexpr int NBAR = 2 * WS + 2 * SB + SA + 2 * ND;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_ABORT = OFF_TMEM + 16;
  static constexpr int SMEM = OFF_ABORT + 16 + 1024;
  static_assert(ND * D_COLS + (SMEM_A ? 0 : SA * A_COLS) <= (int)TMEM_COLS && SA >= 2, "TMEM budget");
  static_assert(!SMEM_A || (MODE != kModeDown && CTAS_PER_SM == 1), "A in shared memory: gate+up / up+activation");
  static_assert(B_PLANE_BYTES % 1024 == 0 && kPairWSlot % 1024 == 0, "TMA tiles stay 1024-byte aligned");
  static_assert(SB >= SA && SB % 2 == 0, "mma_done (odd entries, one commit per two stages) also tracks the A ring");
  static_assert(CTAS_PER_SM * (SMEM + 1024) <= 228 * 1024, "shared memory per SM");
  static_assert(NT % 32 == 0 && NT >= 32 && NT <= 256, "pair MMA with A in tensor memory: N a multiple of 32");
};

}  // namespace

template <int MODE, int NT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, NT > 32 ? 1 : 2)
    grouped_tc_pair_kernel(const TcArgs a, const __grid_constant__ CUtensorMap tm_b0,
                           const __grid_constant__ CUtensorMap tm_b1) {
  using C = PairCfg<MODE, NT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t s_base = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (s_base - raw_base);
  const uint32_t full_w = s_base + C::OFF_BAR;
  const uint32_t empty_w = full_w + 8 * C::WS;
  const uint32_t full_b = empty_w + 8 * C::WS;   // used in the first CTA
  const uint32_t mma_done = full_b + 8 * C::SB;  // both CTAs (multicast commit)
  const uint32_t full_a = mma_done + 8 * C::SB;  // used in the first CTA
  const uint32_t bar_done = full_a + 8 * C::SA;  // [ND], both CTAs (multicast commit)
  const uint32_t bar_dfree = bar_done + 8 * C::ND;  // [ND], used in the first CTA
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  griddep_wait();
  griddep_launch_dependents();
  const int N = (int)a.N, K = (int)a.K;
  const int nst = K / kStageK;
  const int ntile = K / kTileK;
  // Tasks: (active slot, column block of ROWS_PER_PAIR outputs), taken by the
  // pairs in turn.  Both CTAs of a pair, and every role, walk the same list.
  const int ncb = N / C::ROWS_PER_PAIR;
  const int active = min(*a.active_count, (int)a.cap);
  const int ntask = active * ncb;
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  struct Task {
    int e, row_lo, row_hi, n_cta, ngroups;
    bool null_expert;
  };
  auto task = [&](int t) {
    Task k;
    const int slot = t / ncb, cb = t - slot * ncb;
    k.e = a.active_experts[slot];
    k.row_lo = a.offsets[k.e];
    k.row_hi = a.offsets[k.e + 1];
    k.n_cta = cb * C::ROWS_PER_PAIR + (int)rank * (C::ROWS_PER_PAIR / 2);
    k.null_expert = a.packed0[k.e] == nullptr || (MODE == kModeGateUp && a.packed1[k.e] == nullptr);
    k.ngroups = k.null_expert ? 0 : (k.row_hi - k.row_lo + NT - 1) / NT;
    return k;
  };
  // Token rows of pass g of a task: the MMA's N is its rows rounded up to 32;
  // each CTA loads N / 2 of them.
  auto pass_n = [&](const Task& k, int g) -> int {
    const int rows = min(NT, k.row_hi - (k.row_lo + g * NT));
    return (rows + 31) & ~31;
  };

  // ---- set-up: barriers, tensor memory, then both CTAs meet ----
  if (tid == 0) {
    for (int s = 0; s < C::WS; ++s) {
      mbar_init(full_w + 8 * s, 1);
      mbar_init(empty_w + 8 * s, 8);
    }
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(full_b + 8 * s, 1);
      mbar_init(mma_done + 8 * s, 1);
    }
    for (int s = 0; s < C::SA; ++s) mbar_init(full_a + 8 * s, 8);  // 4 decoder warps per stage per CTA
    for (int d = 0; d < C::ND; ++d) {
      mbar_init(bar_done + 8 * d, 1);
      mbar_init(bar_dfree + 8 * d, 8);  // 4 epilogue warps per CTA
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == kPairMmaWarp) {
    tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the first CTA's barriers exist before any remote arrive or TMA signal
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmem_a = tmem + C::ND * C::D_COLS;  // A ring after the D buffers

  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    return false;
  };
  // MMAs of stage x have completed (frees B slot x % SB and A slot x % SA).
  // Stages are committed in pairs: the commit after odd stage x | 1 covers x.
  auto wait_mma = [&](uint32_t x) -> bool {
    x |= 1u;
    return wait(mma_done + 8 * (x % C::SB), (x / C::SB) & 1);
  };

  if (warp == kPairWLoadWarp) {
    // ================= weight tile loader (both CTAs) =================
    if (lane == 0) {
      uint32_t issued = 0;
      for (int t = pair; t < ntask && !*abort_flag; t += npairs) {
        const Task k = task(t);
        if (k.ngroups == 0) continue;
        const CUtensorMap* m = a.wmaps + (size_t)k.e * kMapsPerExpert;
        const CUtensorMap* nib0 = m;
        const CUtensorMap* sc0 = m + 1;
        const CUtensorMap* nib1 = MODE == kModeGateUp ? m + 2 : m;
        const CUtensorMap* sc1 = MODE == kModeGateUp ? m + 3 : m + 1;
        tmap_acquire(nib0);
        tmap_acquire(sc0);
        if (MODE == kModeGateUp) {
          tmap_acquire(nib1);
          tmap_acquire(sc1);
        }
        // Gate+up: 64 gate rows then the same 64 up rows; else 128 rows in two boxes.
        const int y0 = k.n_cta, y1 = MODE == kModeGateUp ? k.n_cta : k.n_cta + kPairWBoxRows;
        for (int g = 0; g < k.ngroups && !*abort_flag; ++g) {
          for (int kt = 0; kt < ntile; ++kt) {
            const uint32_t slot = issued % C::WS, round = issued / C::WS;
            if (round > 0 && !wait(empty_w + 8 * slot, (round - 1) & 1)) break;
            const uint32_t dst = s_base + C::OFF_W + slot * kPairWSlot;
            const uint32_t bar = full_w + 8 * slot;
            mbar_arrive_expect_tx(bar, kPairWSlot);
            tma_load_2d(dst, nib0, kt * (kTileK / 2), y0, bar);
            tma_load_2d(dst + kPairWNib / 2, nib1, kt * (kTileK / 2), y1, bar);
            tma_load_2d(dst + kPairWNib, sc0, kt * (kTileK / 16), y0, bar);
            tma_load_2d(dst + kPairWNib + kPairWBoxRows * 16, sc1, kt * (kTileK / 16), y1, bar);
            ++issued;
          }
        }
      }
      for (uint32_t i = issued > (uint32_t)C::WS ? issued - C::WS : 0; i < issued; ++i)
        mbar_wait(full_w + 8 * (i % C::WS), (i / C::WS) & 1);
    }
  } else if (warp == kPairBLoadWarp) {
    // ================= token tile loader (both CTAs, half each) =================
    if (lane == 0) {
      const uint32_t lead_full_b = mapa_shared(full_b, 0);
      uint32_t issued = 0;
      for (int t = pair; t < ntask && !*abort_flag; t += npairs) {
        const Task k = task(t);
        for (int g = 0; g < k.ngroups && !*abort_flag; ++g) {
          const int half = pass_n(k, g) / 2;
          const int y = k.row_lo + g * NT + (int)rank * half;
          for (int st = 0; st < nst; ++st) {
            const uint32_t slot = issued % C::SB, round = issued / C::SB;
            if (round > 0 && !wait_mma(issued - C::SB)) break;
            const uint32_t dst = s_base + C::OFF_B + slot * C::B_SLOT_BYTES;
            // The first CTA's barrier counts both CTAs' bytes.
            if (rank == 0) mbar_arrive_expect_tx(full_b + 8 * slot, 2 * C::B_SLOT_BYTES);
            tma_load_2d_pair(dst, &tm_b0, st * kStageK, y, lead_full_b + 8 * slot);
            if constexpr (MODE == kModeDown)
              tma_load_2d_pair(dst + C::B_PLANE_BYTES, &tm_b1, st * kStageK, y, lead_full_b + 8 * slot);
            ++issued;
          }
        }
      }
      // The last tiles are consumed by the pair's last MMAs: wait for their
      // completion.  The first CTA also waits for its full_b phases, which
      // count both CTAs' bytes, so no TMA of either CTA still targets its
      // barriers or the peer's shared memory when the pair exits.
      for (uint32_t i = issued > (uint32_t)C::SB ? issued - C::SB : 0; i < issued; ++i) {
        mbar_wait(mma_done + 8 * ((i | 1) % C::SB), ((i | 1) / C::SB) & 1);
        if (rank == 0) mbar_wait(full_b + 8 * (i % C::SB), (i / C::SB) & 1);
      }
    }
  } else if (warp == kPairMmaWarp) {
    // ================= MMA issuer (first CTA) =================
    if (rank == 0 && lane == 0) {
      uint32_t gp = 0, gs = 0;  // passes and stages issued so far (over every task)
      for (int t = pair; t < ntask; t += npairs) {
        const Task k = task(t);
        for (int g = 0; g < k.ngroups; ++g, ++gp, gs += nst) {
          const uint32_t db = gp % C::ND;
          if (gp >= (uint32_t)C::ND) {
            wait(bar_dfree + 8 * db, (gp / C::ND - 1) & 1);  // both epilogues read pass gp - ND
            tc_fence_after();
          }
          const uint32_t idesc = idesc_f16_f32(256, pass_n(k, g));
          const uint32_t dcol = tmem + db * C::D_COLS;
          // Two stages per step: both A stages (each completes only after its
          // token tile has landed too: one decoder lane of this CTA waits for
          // it before arriving), 8 (down: 16) MMAs, one commit, which frees
          // both stages' token slots and A slots.
          for (int st = 0; st < nst; st += 2) {
            const uint32_t ga = gs + st;
            if (!wait(full_a + 8 * (ga % C::SA), (ga / C::SA) & 1)) break;
            if (!wait(full_a + 8 * ((ga + 1) % C::SA), ((ga + 1) / C::SA) & 1)) break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t gx = ga + h;
              const uint32_t bbase = s_base + C::OFF_B + (gx % C::SB) * C::B_SLOT_BYTES;
              const uint32_t abase = C::SMEM_A ? s_base + C::OFF_A + (gx % C::SA) * C::A_STAGE_BYTES
                                               : tmem_a + (gx % C::SA) * C::A_COLS;
#pragma unroll
              for (int s = 0; s < 4; ++s) {
                const uint32_t acc = (st + h > 0 || s > 0) ? 1u : 0u;
                if constexpr (C::SMEM_A)
                  tc_mma_pair_f16_ss(dcol, smem_desc_sw128(abase + s * 32), smem_desc_sw128(bbase + s * 32), idesc, acc);
                else
                  tc_mma_pair_f16_ts(dcol, abase + s * 8, smem_desc_sw128(bbase + s * 32), idesc, acc);
                if constexpr (MODE == kModeDown)
                  tc_mma_pair_f16_ts(dcol, abase + s * 8, smem_desc_sw128(bbase + C::B_PLANE_BYTES + s * 32), idesc,
                                     1u);
              }
            }
            tc_commit_pair(mma_done + 8 * ((ga + 1) % C::SB), 0x3);
          }
          tc_commit_pair(bar_done + 8 * db, 0x3);  // also after a timeout: nothing waits on MMAs in flight
        }
      }
      // No MMA may still run when the tensor memory is freed.
      if (gp > 0) mbar_wait(bar_done + 8 * ((gp - 1) % C::ND), ((gp - 1) / C::ND) & 1);
    }
  } else if (warp < 8) {
    // ================= decoders (both CTAs) =================
    // Warp w decodes TMEM lanes 32 (w % 4) .. + 31 of the stages of parity
    // w / 4, all 64 k of each: two warps per lane quarter alternate stages, so
    // each has two stages of MMA time to decode, store and report one.
    const int q = warp & 3, par = warp >> 2;
    const int L = 32 * q + lane;  // TMEM lane = A row
    const int R = MODE == kModeGateUp ? ((L & 1) ? 64 + (L >> 1) : (L >> 1)) : L;  // row in the weight tile
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const int swz = R & 7;
    const uint32_t lead_full_a = mapa_shared(full_a, 0);
    uint32_t gw = 0;  // weight tiles consumed so far (over every task)
    for (int t = pair; t < ntask; t += npairs) {
      const Task k = task(t);
      for (int g = 0; g < k.ngroups; ++g) {
        for (int kt = 0; kt < ntile; ++kt, ++gw) {
          const uint32_t wslot = gw % C::WS;
          wait(full_w + 8 * wslot, (gw / C::WS) & 1);
          const uint8_t* wtile = smem + C::OFF_W + wslot * kPairWSlot;
          const uint8_t* nrow = wtile + R * 128;
          const uint4 sc4 = *reinterpret_cast<const uint4*>(wtile + kPairWNib + R * 16);
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const int j = 2 * jj + par;  // stage j of the tile (ga has the parity of j)
            const uint32_t ga = gw * 4 + j;
            const uint32_t aslot = ga % C::SA;
            // k 64 j .. + 63 of this row: 16-byte chunks 2 j and 2 j + 1 (swizzled), four block scales.
            const uint4 q0 = *reinterpret_cast<const uint4*>(nrow + (((2 * j) ^ swz) << 4));
            const uint4 q1 = *reinterpret_cast<const uint4*>(nrow + (((2 * j + 1) ^ swz) << 4));
            uint32_t sclo, schi;  // f16x2 of scale bytes (4 j, 4 j + 1) and (4 j + 2, 4 j + 3)
            e4m3x4_to_f16x2x2(par ? (jj ? sc4.w : sc4.y) : (jj ? sc4.z : sc4.x), sclo, schi);
            uint32_t v[32];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 qv = h == 0 ? q0 : q1;
              const uint32_t sc = h == 0 ? sclo : schi;
              const uint32_t wv[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint32_t scl = i < 2 ? bcast_lo(sc) : bcast_hi(sc);
                uint32_t dec[4];
                e2m1x8_to_f16x2x4(wv[i], dec);
#pragma unroll
                for (int m = 0; m < 4; ++m) v[16 * h + i * 4 + m] = hmul2_u32(dec[m], scl);
              }
            }
            if (jj == 1) {  // this warp's last stage of the weight tile
              __syncwarp();
              if (lane == 0) mbar_arrive(empty_w + 8 * wslot);
            }
            if (ga >= (uint32_t)C::SA) wait_mma(ga - C::SA);  // the A slot's previous MMAs are done
            if constexpr (C::SMEM_A) {
              // Row L of the stage's K-major tile, 128-byte swizzle: 16-byte
              // chunk c (k 8 c .. 8 c + 7) at chunk position c ^ (L % 8).
              uint8_t* arow = smem + C::OFF_A + aslot * C::A_STAGE_BYTES + L * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(arow + ((c ^ (L & 7)) << 4)) =
                    make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
              fence_proxy_async_smem();  // generic-proxy writes -> the MMA's async-proxy reads
            } else {
              tc_fence_after();
              tmem_st32(tmem_a + lane_off + aslot * C::A_COLS, v);
              tmem_wait_st();
              tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) {
              // In the first CTA, warp 0 / 4 also reports the stage's token tile.
              if (rank == 0 && q == 0) wait(full_b + 8 * (ga % C::SB), (ga / C::SB) & 1);
              mbar_arrive_remote(lead_full_a + 8 * aslot);
            }
          }
        }
      }
    }
  } else if (warp >= kPairEpiWarp0) {
    // ================= epilogue (both CTAs) =================
    const int q = warp & 3;
    const int L = 32 * q + lane;
    const int et = tid - 32 * kPairEpiWarp0;  // 0 .. 127
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const uint32_t lead_dfree = mapa_shared(bar_dfree, 0);
    const int odd = lane & 1;
    uint32_t gp = 0;  // passes drained so far (over every task)
    for (int t = pair; t < ntask; t += npairs) {
      const Task k = task(t);
      if (k.null_expert) {
        // NULL expert: this CTA's outputs of its rows are zero.
        constexpr int W = C::ROWS_PER_PAIR / 2;
        for (int i = et; i < (k.row_hi - k.row_lo) * W; i += 128)
          a.out[(size_t)(k.row_lo + i / W) * N + k.n_cta + i % W] = 0.0f;
        continue;
      }
      const float s2a = a.s2_0[k.e];
      const float s2b = a.s2_1[k.e];
      // Output n of this lane: gate+up pairs lanes (2j: gate, 2j + 1: up of n_cta + j).
      const int n = MODE == kModeGateUp ? k.n_cta + (L >> 1) : k.n_cta + L;
      for (int g = 0; g < k.ngroups; ++g, ++gp) {
        const uint32_t db = gp % C::ND;
        const int g0 = k.row_lo + g * NT;
        const int nrows = min(NT, k.row_hi - g0);
        bool ok = wait(bar_done + 8 * db, (gp / C::ND) & 1);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        const uint32_t dcol = tmem + lane_off + db * C::D_COLS;
#pragma unroll 1
        for (int c0 = 0; c0 < nrows; c0 += 32) {
          // lane l holds the activation-row scale of token c0 + l
          const float xm_l = (c0 + lane < nrows) ? a.bexp[g0 + c0 + lane] : 0.0f;
          // 32 columns per wait (the D buffer holds NT >= c0 + 32 columns).
          uint32_t d[32];
#pragma unroll
          for (int h = 0; h < 4; ++h) tmem_ld8(dcol + c0 + 8 * h, *reinterpret_cast<uint32_t(*)[8]>(d + 8 * h));
          tmem_wait_ld();
          if constexpr (MODE == kModeGateUp) {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              // Even lane: gate of tokens t, t + 1; odd lane: up of the same.
              // After the swap the even lane holds (g, u) of token t, the odd
              // lane (g, u) of token t + 1.
              const float mine0 = __uint_as_float(d[j]), mine1 = __uint_as_float(d[j + 1]);
              const float other = __shfl_xor_sync(0xffffffffu, odd ? mine0 : mine1, 1);
              const float gv = odd ? other : mine0;
              const float uv = odd ? mine1 : other;
              const int tl = j + odd;
              const float xm = __shfl_sync(0xffffffffu, xm_l, tl);
              const int tt = c0 + tl;
              if (ok && tt < nrows) a.out[(size_t)(g0 + tt) * N + n] = silu_f32(gv * xm * s2a) * (uv * xm * s2b);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float xm = __shfl_sync(0xffffffffu, xm_l, j);
              const int tt = c0 + j;
              float v = __uint_as_float(d[j]) * xm * s2a;
              if constexpr (MODE == kModeUpAct) v = activation_f32(a.activation, v);
              if (ok && tt < nrows) a.out[(size_t)(g0 + tt) * N + n] = v;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(lead_dfree + 8 * db);
      }
    }
  }

  __syncthreads();
  __syncwarp();
  cluster_sync();  // no more remote arrives, and the pair's MMAs are done
  if (warp == kPairMmaWarp) {
    __syncwarp();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

namespace {

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 2) return 148;
  return n;
}

// Persistent launch: one pair per two SMs (two at 32-row passes), or fewer
// when there are fewer tasks than that.
template <int MODE, int NT>
cudaError_t launch_tc_pair_impl(const TcArgs& a, const CUtensorMap& b0, const CUtensorMap& b1, uint32_t cap,
                                cudaStream_t stream) {
  using C = PairCfg<MODE, NT>;
  auto kern = grouped_tc_pair_kernel<MODE, NT>;
  cudaError_t err = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::SMEM);
  if (err != cudaSuccess) return err;
  const uint64_t tasks = (uint64_t)cap * (a.N / C::ROWS_PER_PAIR);
  uint64_t pairs = (uint64_t)(sm_count() / 2) * C::CTAS_PER_SM;
  if (pairs > tasks) pairs = tasks;
  if (pairs == 0) return cudaSuccess;
  TcArgs args = a;
  args.cap = cap;
  return launch_pdl(kern, dim3((unsigned)(2 * pairs)), dim3(kPairThreads), C::SMEM, stream, args, b0, b1);
}

}  // namespace
