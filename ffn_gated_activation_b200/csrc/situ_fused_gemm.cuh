// Grouped GEMMs on the sm_100a tensor cores with a SiTU-GLU epilogue: the
// fused FC1 forward and the fused FC2 data gradient.
//
// FC1 (Megatron-LM PR #6673, "Design": with a SiTU-capable cuDNN frontend,
// FC1's grouped GEMM and the SiTU-GLU activation run as one operation).  For a
// token row r routed to expert e,
//     G[r, i] = sum_k X[r, k] W1_e[i, k],  U[r, i] = sum_k X[r, k] W1_e[I + i, k]
//     Y[r, i] = T_g(G) T_u(U) w[r]
// FC2 data gradient with the SiTU-GLU backward (the "dSiTU" of the fused
// grouped MLP's backward, Megatron-LM PR #6673, "Test results"):
//     dY[r, i] = sum_h dOut[r, h] W2_e[h, i]   (W2 passed transposed: W2T_e [I, H])
//     dG = dY w T_u T_g',  dU = dY w T_g T_u',  d_w[r] = sum_i dY T_g T_u
// The fp32 accumulators never leave the chip: G and U (or dY) are never
// written, only Y (or dG, dU and per-tile d_w partials).
//
// Included into situ_glu.cu (anonymous namespace): it uses the library's
// element arithmetic (fwd_pair_abs, bwd_pair), storage helpers and bounded
// mbarriers.
//
// Structure (one CTA per SM, persistent over output tiles):
//   * a tile is 128 token rows; its B operand is 256 rows of the expert's
//     weight, so one tcgen05.mma (M = 128, N = 256, K = 16) per 16 hidden
//     elements fills 256 TMEM columns.  FC1 puts gate columns [n0, n0 + 128)
//     and the matching up columns side by side (128 output columns per tile);
//     FC2 takes 256 consecutive dY columns;
//   * warp 0 streams 64-wide K slices with TMA (128-byte swizzle) into a
//     4-stage shared-memory ring; warp 1 owns the TMEM allocation and issues
//     the MMAs from one lane, releasing each stage with tcgen05.commit;
//   * two TMEM accumulators (512 columns) let warps 2-5 run the epilogue of
//     one tile while the next tile's MMAs run: each epilogue thread owns one
//     accumulator row (its warp's TMEM lane quarter), reads it with
//     tcgen05.ld, applies the element arithmetic in fp32 and stores bf16;
//   * tiles are numbered expert by expert from device-side row offsets; within
//     an expert, groups of kGroupM row tiles sweep the column tiles so that
//     the CTAs running together share operand tiles in L2.
// Every wait is bounded (kWaitLimitNs); a wait that expires sets the device
// status word and a CTA-wide abort flag, every role then stops issuing work,
// the producer waits (bounded) for its own copies, the MMA warp for its own
// MMAs, and TMEM is freed.
//
// The library launches the two-SM form at the end of this file (clusters of
// two CTAs sharing 256-row tiles through tcgen05 cta_group::2) whenever the
// device can hold such clusters, and this one-SM kernel otherwise.

namespace fc1 {

constexpr int kBM = 128;                   // token rows per tile (UMMA M)
constexpr int kBN = 128;                   // output columns per tile
constexpr int kUmmaN = 2 * kBN;            // gate + up accumulator columns (UMMA N)
constexpr int kBK = 64;                    // hidden elements per stage: one 128-byte swizzle row
constexpr int kUmmaK = 16;                 // K of one tcgen05.mma.kind::f16
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;     // 16 KiB
constexpr int kBHalfBytes = kBN * kBK * 2; // 16 KiB (gate rows, then up rows)
constexpr int kStageBytes = kABytes + 2 * kBHalfBytes;
constexpr int kAccCols = kUmmaN;           // fp32 TMEM columns per accumulator
constexpr int kAccBufs = 2;
constexpr int kTmemCols = kAccCols * kAccBufs;  // 512: the whole TMEM of the SM
constexpr int kThreads = 192;              // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kEpiThreads = 128;
#ifndef SITU_FC1_GROUP_M
#define SITU_FC1_GROUP_M 8
#endif
constexpr int kGroupM = SITU_FC1_GROUP_M;  // row tiles that sweep the column tiles together
constexpr int kMaxExperts = 1024;
// Header after the ring: 12 mbarriers, TMEM base and abort flag, the drain
// mbarrier; then per-expert tables (row ranges, first tile).
constexpr int kHeaderBytes = 128;

// Instruction descriptor of tcgen05.mma.kind::f16: fp32 accumulator (bits
// 4-5 = 1), bf16 A and B (bits 7-9, 10-12 = 1), both K-major (bits 15, 16 =
// 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kUmmaN >> 3) << 17) |
                            (static_cast<uint32_t>(kBM >> 4) << 24);

// The epilogues' global accesses (plain, L1-cached: measured faster here than
// the streaming forms).
__device__ __forceinline__ uint4 epi_ld(const char* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void epi_st(char* p, const uint4& v) { *reinterpret_cast<uint4*>(p) = v; }

struct Args {
  const int64_t* offsets;  // device [experts + 1]
  int experts;
  int64_t tokens;
  int hidden;
  int inter;
  RwArgs rw;
  char* y;                 // FC1: Y bf16 [tokens, >= inter]; FC2: d_gate_up bf16 [tokens, >= 2 inter]
  int64_t y_pitch;         // bytes
  const char* gate_up;     // FC2: the saved gate_up bf16 [tokens, >= 2 inter]
  int64_t gu_pitch;        // bytes
  float* partials;         // FC2: d_w partials [tokens][inter / 256] (NULL: not wanted)
  Coeffs c;
};

// Shared-memory matrix descriptor of a K-major tile in the 128-byte swizzle
// layout TMA writes: rows of 128 bytes, 8-row groups 1024 bytes apart (stride
// byte offset), start address in 16-byte units, descriptor version 1 (bits
// 46-47), layout type 2 = 128-byte swizzle (bits 61-63).  The leading byte
// offset is unused for swizzled K-major tiles and set to 1 (16 bytes).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t smem_addr) {
  uint64_t d = static_cast<uint64_t>((smem_addr >> 4) & 0x3fffu);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t x, int32_t y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D (TMEM) (+)= A (smem) B (smem)^T; accumulate = 0 overwrites D.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// The wait, with the loaded registers passed through it: their uses cannot be
// scheduled above the point where the asynchronous load has landed.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16], uint32_t (&q)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                 "+r"(q[0]), "+r"(q[1]), "+r"(q[2]), "+r"(q[3]), "+r"(q[4]), "+r"(q[5]), "+r"(q[6]), "+r"(q[7]),
                 "+r"(q[8]), "+r"(q[9]), "+r"(q[10]), "+r"(q[11]), "+r"(q[12]), "+r"(q[13]), "+r"(q[14]), "+r"(q[15])
               :
               : "memory");
}

// Bounded wait that also gives up once another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicExch(&g_device_status, kStatusWaitExpired);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// A tile of the grouped problem.
struct Tile {
  int expert;
  int64_t m0;    // first token row
  int64_t m_end; // one past the expert's last row
  int n0;        // first output column
};

// Tile t (numbered expert by expert; inside an expert, groups of kGroupM row
// tiles of BM rows sweep all column tiles).  first_tile[e] is the first tile
// of expert e, first_tile[experts] the total; [lo[e], hi[e]) its rows.
template <int BM = kBM>
__device__ __forceinline__ Tile decode_tile(int t, const int* first_tile, const int64_t* lo, const int64_t* hi,
                                            int experts, int n_tiles, int out_cols) {
  int left = 0, right = experts - 1;  // the last e with first_tile[e] <= t
  while (left < right) {
    const int mid = (left + right + 1) >> 1;
    if (first_tile[mid] <= t) left = mid; else right = mid - 1;
  }
  const int e = left;
  const int local = t - first_tile[e];
  const int64_t r0 = lo[e], r1 = hi[e];
  const int m_tiles = static_cast<int>((r1 - r0 + BM - 1) / BM);
  const int group = local / (kGroupM * n_tiles);
  const int first_m = group * kGroupM;
  const int group_m = min(kGroupM, m_tiles - first_m);
  const int within = local - group * kGroupM * n_tiles;
  Tile tile;
  tile.expert = e;
  tile.m0 = r0 + static_cast<int64_t>(first_m + within % group_m) * BM;
  tile.m_end = r1;
  tile.n0 = (within / group_m) * out_cols;
  return tile;
}

// Row range [lo_e, hi_e) of each expert (offsets clamped to [0, tokens], a
// decreasing pair read as empty) and its first tile of BM rows: lane l of the
// calling warp takes a contiguous run of experts, a warp scan adds the runs'
// tile counts.
template <int BM>
__device__ __forceinline__ void scan_experts(const Args& a, int n_tiles, int lane, int64_t* lo, int64_t* hi,
                                             int* first_tile) {
  const int per = (a.experts + 31) / 32;
  const int e0 = min(a.experts, lane * per), e1 = min(a.experts, e0 + per);
  int count = 0;
  for (int e = e0; e < e1; ++e) {
    int64_t r0 = a.offsets[e], r1 = a.offsets[e + 1];
    r0 = r0 < 0 ? 0 : (r0 > a.tokens ? a.tokens : r0);
    r1 = r1 < r0 ? r0 : (r1 > a.tokens ? a.tokens : r1);
    lo[e] = r0;
    hi[e] = r1;
    count += static_cast<int>((r1 - r0 + BM - 1) / BM) * n_tiles;
  }
  int incl = count;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - count;
  for (int e = e0; e < e1; ++e) {
    first_tile[e] = run;
    run += static_cast<int>((hi[e] - lo[e] + BM - 1) / BM) * n_tiles;
  }
  if (lane == 31) first_tile[a.experts] = incl;
}

// FC1: B = the expert's gate rows [n0, n0 + 128) then its up rows; the
// epilogue turns gate column c and up column 128 + c into Y column n0 + c.
struct Fc1Epilogue {
  static constexpr int kOutCols = kBN;
  __device__ __forceinline__ static void b_rows(const Args& a, const Tile& t, int32_t& r0, int32_t& r1) {
    r0 = t.expert * 2 * a.inter + t.n0;
    r1 = r0 + a.inter;
  }
  template <int GATE, bool HAS_LB>
  __device__ __forceinline__ static void run(const Args& a, const Tile& tile, int64_t row, bool valid,
                                             uint32_t taddr) {
    const float wbb = (valid ? load_rw(a.rw, row) : 0.0f) * a.c.bb;
    char* yrow = a.y + (valid ? row : 0) * a.y_pitch + static_cast<int64_t>(tile.n0) * 2;
#pragma unroll 1
    for (int c = 0; c < kBN; c += 16) {
      uint32_t g[16], u[16];
      tmem_ld16(taddr + c, g);
      tmem_ld16(taddr + kBN + c, u);
      tmem_ld_wait(g, u);
      uint32_t q[8];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 gv = make_uint4(g[4 * v], g[4 * v + 1], g[4 * v + 2], g[4 * v + 3]);
        const uint4 uv = make_uint4(u[4 * v], u[4 * v + 1], u[4 * v + 2], u[4 * v + 3]);
#pragma unroll
        for (int p = 0; p < 2; ++p)
          q[2 * v + p] =
              Bf16::pack(fwd_pair_abs<GATE, HAS_LB, F32>(F32::pair(gv, p), F32::pair(uv, p), splat(wbb), a.c));
      }
      if (valid) {
        epi_st(yrow + c * 2, make_uint4(q[0], q[1], q[2], q[3]));
        epi_st(yrow + c * 2 + 16, make_uint4(q[4], q[5], q[6], q[7]));
      }
    }
  }
};

// FC2 data gradient: B = the expert's transposed FC2 rows [n0, n0 + 256); the
// epilogue reads G, U of the saved gate_up row, writes dG, dU for columns
// [n0, n0 + 256) and the tile's share of d_w.
struct Fc2Epilogue {
  static constexpr int kOutCols = kUmmaN;
  __device__ __forceinline__ static void b_rows(const Args& a, const Tile& t, int32_t& r0, int32_t& r1) {
    r0 = t.expert * a.inter + t.n0;
    r1 = r0 + kBN;
  }
  template <int GATE, bool HAS_LB>
  __device__ __forceinline__ static void run(const Args& a, const Tile& tile, int64_t row, bool valid,
                                             uint32_t taddr) {
    const float w = valid ? load_rw(a.rw, row) : 0.0f;
    const float2 k = bwd_row_consts<HAS_LB>(w, a.c);
    const float2 kdg = splat(k.x), kdu = splat(k.y);
    const int64_t r = valid ? row : 0;
    const char* grow = a.gate_up + r * a.gu_pitch + static_cast<int64_t>(tile.n0) * 2;
    const char* urow = grow + static_cast<int64_t>(a.inter) * 2;
    char* dgrow = a.y + r * a.y_pitch + static_cast<int64_t>(tile.n0) * 2;
    char* durow = dgrow + static_cast<int64_t>(a.inter) * 2;
    float2 acc = make_float2(0.0f, 0.0f);
    // Chunk c + 16's accumulator columns (TMEM) and saved gate_up values
    // (global) are requested before chunk c is computed, so their latency
    // overlaps the arithmetic: this warp is alone on its scheduler.
    uint32_t d[16];
    uint4 gn[2], un[2];
    tmem_ld16(taddr, d);
    if (valid) {
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        gn[v] = epi_ld(grow + v * 16);
        un[v] = epi_ld(urow + v * 16);
      }
    }
#pragma unroll 1
    for (int c = 0; c < kUmmaN; c += 16) {
      tmem_ld_wait(d);
      uint32_t dc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) dc[i] = d[i];
      const uint4 gc[2] = {gn[0], gn[1]}, uc[2] = {un[0], un[1]};
      if (c + 16 < kUmmaN) {  // uniform over the warp
        tmem_ld16(taddr + c + 16, d);
        if (valid) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            gn[v] = epi_ld(grow + (c + 16) * 2 + v * 16);
            un[v] = epi_ld(urow + (c + 16) * 2 + v * 16);
          }
        }
      }
      if (valid) {
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const uint4 gv = gc[v], uv = uc[v];
          uint4 dgv, duv;
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            float2 dg, du;
            const float2 go = make_float2(__uint_as_float(dc[8 * v + 2 * p]), __uint_as_float(dc[8 * v + 2 * p + 1]));
            bwd_pair<GATE, HAS_LB, Bf16, true>(Bf16::pair(gv, p), Bf16::pair(uv, p), go, kdg, kdu, a.c, dg, du, acc);
            Bf16::put(dgv, p, dg);
            Bf16::put(duv, p, du);
          }
          epi_st(dgrow + c * 2 + v * 16, dgv);
          epi_st(durow + c * 2 + v * 16, duv);
        }
      }
    }
    if (valid && a.partials != nullptr)
      a.partials[row * (a.inter / kUmmaN) + tile.n0 / kUmmaN] = (acc.x + acc.y) * bwd_dw_scale(a.c);
  }
};

template <class Epi, int GATE, bool HAS_LB>
__global__ void __launch_bounds__(kThreads, 1)
    situ_fused_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                           const Args a) {
  extern __shared__ unsigned char smem_raw[];
  // The ring needs 1024-byte alignment (128-byte swizzle atoms of 8 rows).
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + kAccBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* drain = acc_empty + kAccBufs + 1;  // after the TMEM slot and the abort flag
  int64_t* lo = reinterpret_cast<int64_t*>(smem + kStages * kStageBytes + kHeaderBytes);  // [experts]
  int64_t* hi = lo + a.experts;                                                          // [experts]
  int* first_tile = reinterpret_cast<int*>(hi + a.experts);                              // [experts + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = a.inter / Epi::kOutCols;
  const int k_blocks = a.hidden / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiThreads);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) scan_experts<kBM>(a, n_tiles, lane, lo, hi, first_tile);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = first_tile[a.experts];

  if (warp == 0) {
    // ---- TMA producer ----
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0;  // bit s: stage s holds a copy that may still be in flight
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
      const Tile tile = decode_tile(t, first_tile, lo, hi, a.experts, n_tiles, Epi::kOutCols);
      int32_t wrow0, wrow1;
      Epi::b_rows(a, tile, wrow0, wrow1);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!wait_or_abort(&empty[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          unsigned char* st = ring + stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_2d(st, &tmap_x, kb * kBK, static_cast<int32_t>(tile.m0), &full[stage]);
          tma_load_2d(st + kABytes, &tmap_w, kb * kBK, wrow0, &full[stage]);
          tma_load_2d(st + kABytes + kBHalfBytes, &tmap_w, kb * kBK, wrow1, &full[stage]);
        }
        __syncwarp();
        issued |= 1u << stage;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      // Aborted: let the copies this warp issued land before the CTA exits.
      // Stage s's latest copy completes the phase that the MMA warp waits for;
      // wait for it (bounded) without the abort shortcut.
      for (int s = 0; s < kStages; ++s) {
        if (!(issued & (1u << s))) continue;
        const uint32_t ph = (s < stage) ? phase : (phase ^ 1u);  // phase of stage s's latest fill
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait(&full[s], ph) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    int stage = 0;
    uint32_t phase = 0;
    uint32_t acc_phase = 0;  // bit b: phase of accumulator b
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x, ++it) {
      const int b = it & 1;
      if (!wait_or_abort(&acc_empty[b], ((acc_phase >> b) & 1u) ^ 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kAccCols);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!wait_or_abort(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(ring + stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            umma_bf16(d_tmem, smem_desc_sw128(a_addr + kk * kUmmaK * 2), smem_desc_sw128(b_addr + kk * kUmmaK * 2),
                      (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);  // the stage is free once these MMAs have read it
        }
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&acc_full[b]);  // the accumulator is complete
      __syncwarp();
      acc_phase ^= 1u << b;
    }
    if (!ok || *abort_flag) {
      // Aborted: wait (bounded) until every MMA this warp issued is done
      // before TMEM is freed.
      if (lane == 0) umma_commit(drain);
      __syncwarp();
      const unsigned long long t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    // ---- epilogue: warps 2-5, one accumulator row per thread ----
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row_in_tile = quarter * 32 + lane;
    uint32_t acc_phase = 0;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const int b = it & 1;
      if (!wait_or_abort(&acc_full[b], (acc_phase >> b) & 1u, abort_flag)) break;
      tc_fence_after();
      const Tile tile = decode_tile(t, first_tile, lo, hi, a.experts, n_tiles, Epi::kOutCols);
      const int64_t row = tile.m0 + row_in_tile;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * kAccCols);
      Epi::template run<GATE, HAS_LB>(a, tile, row, row < tile.m_end, taddr);
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
      acc_phase ^= 1u << b;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols) : "memory");
}

// ---- Two-SM form (tcgen05 cta_group::2) ---------------------------------------
// A cluster of two CTAs on two SMs computes a 256-row tile: CTA r of the pair
// stages token rows [m0 + 128 r, m0 + 128 r + 128) of A and half of B (FC1:
// the gate rows for r = 0, the up rows for r = 1; FC2: B rows [n0 + 128 r,
// n0 + 128 r + 128)) in its own shared memory, and one thread of CTA 0 issues
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16), which reads both CTAs'
// halves and leaves each CTA's 128 accumulator rows (all 256 columns) in that
// CTA's TMEM.  Each SM so reads half of B per K slice instead of all of it:
// a third fewer operand bytes per FLOP from L2.  The epilogue is the one-SM
// kernel's, per CTA.  No load is multicast: every CTA loads its own tiles,
// whose completion bytes both count on CTA 0's stage barrier (the loads'
// cta_group::2 form), and CTA 0's MMA commits arrive on both CTAs' barriers.
constexpr int kBM2 = 2 * kBM;                      // token rows per cluster tile
#ifndef SITU_FC2SM_STAGES
#define SITU_FC2SM_STAGES 6
#endif
constexpr int kStages2 = SITU_FC2SM_STAGES;
constexpr int kStageBytes2 = kABytes + kBHalfBytes;  // 32 KiB per CTA
// Header after the ring: 17 mbarriers, the TMEM base and the abort flag; then
// the per-expert tables.
constexpr int kHeaderBytes2 = 256;
// kind::f16, fp32 accumulator, bf16 A and B, K-major, N = 256, M = 256.
constexpr uint32_t kIdesc2 = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kUmmaN >> 3) << 17) |
                             (static_cast<uint32_t>(kBM2 >> 4) << 24);

// Arrive on an mbarrier of either CTA of the cluster (shared::cluster address).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's shared memory whose completion bytes count on the
// mbarrier at `bar` (a shared::cluster address; here CTA 0's).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int32_t x, int32_t y,
                                                 uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8, %9, %10, %11, %12}, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc2), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u),
      "r"(0u), "r"(0u));
}
// Arrive on the mbarrier at this offset in both CTAs once every MMA issued so
// far by this thread is done.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}
// Arrive on this CTA's own mbarrier once this thread's MMAs are done.
__device__ __forceinline__ void umma_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool wait_or_abort_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicExch(&g_device_status, kStatusWaitExpired);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

static_assert((2 * kStages2 + 4 * kAccBufs / 2 + 1) * 8 + 8 <= kHeaderBytes2, "2-SM header overflows");

template <class Epi, int GATE, bool HAS_LB>
__global__ void __launch_bounds__(kThreads, 1)
    situ_fused_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                               const Args a) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  unsigned char* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  unsigned char* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages2 * kStageBytes2);
  uint64_t* empty = full + kStages2;
  uint64_t* acc_full = empty + kStages2;
  uint64_t* acc_empty = acc_full + kAccBufs;
  uint64_t* drain = acc_empty + kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int64_t* lo = reinterpret_cast<int64_t*>(smem + kStages2 * kStageBytes2 + kHeaderBytes2);  // [experts]
  int64_t* hi = lo + a.experts;                                                            // [experts]
  int* first_tile = reinterpret_cast<int*>(hi + a.experts);                                // [experts + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int cl = static_cast<int>(cluster_index()), ncl = static_cast<int>(cluster_count());
  const int n_tiles = a.inter / Epi::kOutCols;
  const int k_blocks = a.hidden / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(&full[s], 1);   // CTA 0's producer arrives; both CTAs' copies add bytes
      mbar_init(&empty[s], 1);  // CTA 0's MMA commit
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);                 // CTA 0's MMA commit
      mbar_init(&acc_empty[b], 2 * kEpiThreads);  // every epilogue thread of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) scan_experts<kBM2>(a, n_tiles, lane, lo, hi, first_tile);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = first_tile[a.experts];

  if (warp == 0) {
    // ---- TMA producer (both CTAs) ----
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0;
    bool ok = true;
    for (int t = cl; ok && t < total; t += ncl) {
      const Tile tile = decode_tile<kBM2>(t, first_tile, lo, hi, a.experts, n_tiles, Epi::kOutCols);
      int32_t wrow0, wrow1;
      Epi::b_rows(a, tile, wrow0, wrow1);
      const int32_t wrow = leader ? wrow0 : wrow1;
      const int32_t arow = static_cast<int32_t>(tile.m0 + static_cast<int64_t>(rank) * kBM);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!wait_or_abort_cluster(&empty[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          unsigned char* st = ring + stage * kStageBytes2;
          const uint32_t bar = peer_addr(&full[stage], 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes2);
          tma_load_2d_pair(st, &tmap_x, kb * kBK, arow, bar);
          tma_load_2d_pair(st + kABytes, &tmap_w, kb * kBK, wrow, bar);
        }
        __syncwarp();
        issued |= 1u << stage;
        if (++stage == kStages2) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && leader) {
      // Aborted: let the copies of both CTAs land (they count on CTA 0's
      // barriers) before the cluster exits; bounded.
      for (int s = 0; s < kStages2; ++s) {
        if (!(issued & (1u << s))) continue;
        const uint32_t ph = (s < stage) ? phase : (phase ^ 1u);
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait_cluster(&full[s], ph) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ---- MMA issuer (CTA 0 only) ----
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = cl; ok && t < total; t += ncl, ++it) {
        const int b = it & 1;
        if (!wait_or_abort_cluster(&acc_empty[b], ((acc_phase >> b) & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kAccCols);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!wait_or_abort_cluster(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_addr = smem_u32(ring + stage * kStageBytes2);
            const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
            for (int kk = 0; kk < kBK / kUmmaK; ++kk)
              umma_bf16_pair(d_tmem, smem_desc_sw128(a_addr + kk * kUmmaK * 2),
                             smem_desc_sw128(b_addr + kk * kUmmaK * 2), (kb | kk) != 0 ? 1u : 0u);
            umma_commit_pair(&empty[stage]);  // both CTAs' stage is free once these MMAs have read it
          }
          __syncwarp();
          if (++stage == kStages2) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_pair(&acc_full[b]);  // both CTAs' accumulator rows are complete
        __syncwarp();
        acc_phase ^= 1u << b;
      }
      if (!ok || *abort_flag) {
        if (lane == 0) umma_commit_pair_local(drain);
        __syncwarp();
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait_cluster(drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ---- epilogue: warps 2-5 of both CTAs, one accumulator row per thread ----
    const int quarter = warp & 3;
    const int row_in_tile = static_cast<int>(rank) * kBM + quarter * 32 + lane;
    uint32_t acc_phase = 0;
    int it = 0;
    for (int t = cl; t < total; t += ncl, ++it) {
      const int b = it & 1;
      if (!wait_or_abort_cluster(&acc_full[b], (acc_phase >> b) & 1u, abort_flag)) break;
      tc_fence_after();
      const Tile tile = decode_tile<kBM2>(t, first_tile, lo, hi, a.experts, n_tiles, Epi::kOutCols);
      const int64_t row = tile.m0 + row_in_tile;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * kAccCols);
      Epi::template run<GATE, HAS_LB>(a, tile, row, row < tile.m_end, taddr);
      tc_fence_before();
      mbar_arrive_remote(peer_addr(&acc_empty[b], 0));
      acc_phase ^= 1u << b;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or copies may touch its memory
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols) : "memory");
}

}  // namespace fc1
