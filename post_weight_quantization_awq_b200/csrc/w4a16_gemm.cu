// W4A16 GEMM on the packed output of the search: the step after the path,
// in which a layer's fp16 activations meet its 4-bit weights ("05 — AWQ:
// Activation-Aware Weight Scaling" §5: qweight [in, out/8] int32 with output o
// in nibble o % 8, qzeros [in/g, out/8], scales fp16 [in/g, out]; "AWQ and
// Activation-Aware Scaling" / the papermap summary: the weights are
// dequantised on the fly inside the GEMM).
//
//   Y[t][o] = RN16( sum_j X[t][j] * Wd[o][j] ),  Wd[o][j] = RN16((q - z) * scale)
//
// with q = the code of (o, j), z the zero of (o, j/g), scale = scales[j/g][o]:
// the fp16 weights a consumer multiplies.  fp32 accumulation on the tensor
// cores.
//
// sm_100a design, one CTA per SM (448 threads), persistent over 256 x 256
// output tiles (two M = 128 accumulators share every dequantised B tile, which
// halves the conversion work per flop):
//   warp 0      TMA loads of the 256 x 64 X tile (K-major, 128-byte swizzle)
//               and of the 64 x 32 block of packed words behind the B tile;
//   warps 6..13 dequantise the 64 x 256 weight tile: each thread turns int32
//               words (8 outputs of one input channel each) into 16-byte
//               chunks of an MN-major 128-byte-swizzled B tile — the packed
//               layout is input-major, which is exactly MN-major for B, so no
//               transpose is needed.  Within a chunk the outputs sit in the
//               order 0,4,1,5,2,6,3,7 (what two mask operations per pair give);
//               the accumulator columns carry the same order and the epilogue
//               puts them back when it packs Y.  The words come from shared
//               memory (staged by TMA with the X tile), zero points and
//               scales from L1/L2 one step ahead;
//   warp 1      one thread issues tcgen05.mma kind::f16 (M = 128, N = 256,
//               K = 16), two per K step, into the two halves of TMEM;
//   warps 2..5  read the accumulators (tcgen05.ld), round to fp16 and store Y
//               (the next tile's MMAs wait for them: TMEM holds one tile).
// Three pipeline stages of (32 + 32 + 8) KiB.  Every mbarrier wait is bounded; on a
// timeout the CTA records kDevTimeout, drains its copies and MMAs, frees TMEM
// and exits.
#include <cuda.h>
#include <cuda_fp16.h>

#include "awq_launch.h"

namespace awq {

namespace {
constexpr int QBM = 256, QMM = 128, QBN = 256, QBK = 64, QSTAGES = 3;  // CTA rows, MMA rows
constexpr int QW_STAGES = 4;  // packed-word stages: their own ring, refilled as soon as read
constexpr uint32_t QA_BYTES = QBM * QBK * 2;   // 32 KiB
constexpr uint32_t QA_HALF = QMM * QBK * 2;    // rows 128..255 of the X tile start here
constexpr uint32_t QB_BOX = QBK * 128;         // 64 input channels x 64 outputs (8 KiB)
constexpr uint32_t QB_BYTES = 4 * QB_BOX;      // 32 KiB
constexpr uint32_t QW_BYTES = QBK * (QBN / 8) * 4;  // packed words of a B tile (8 KiB)
constexpr uint32_t QTMEM_COLS = 512;
constexpr int QGROUP_M = 16;
constexpr int QW_WPROD = 6;                    // the packed words' TMA producer
constexpr int QW_DEQ = 7;                      // first dequantising warp
constexpr int QN_DEQ = 8;                      // dequantising warps (two per sub-partition)
constexpr int Q_WORDS = QBK * (QBN / 8) / (QN_DEQ * 32);  // words per thread per K tile (8)
constexpr int Q_THREADS = (QW_DEQ + QN_DEQ) * 32;         // 480: up to 136 registers
static_assert(QN_DEQ % 8 == 0 && Q_WORDS % 2 == 0 && QN_DEQ * Q_WORDS == QBK, "dequant split");
constexpr uint32_t Q_DRAIN = 1u << 22;
// kind::f16, fp16 A/B, fp32 D, A K-major, B MN-major, N = 256, M = 128
constexpr uint32_t IDESC_Q = (1u << 4) | (1u << 16) | ((uint32_t)(QBN >> 3) << 17) |
                             ((uint32_t)(QMM >> 4) << 24);

struct __align__(8) QTail {
  uint64_t ld[QSTAGES];       // TMA bytes of the X tile
  uint64_t full[QSTAGES];     // the B tile: one arrival per dequantising warp
  uint64_t empty[QSTAGES];    // MMA commit: X and B of the stage are free
  uint64_t wld[QW_STAGES];    // TMA bytes of the packed words
  uint64_t wempty[QW_STAGES]; // words read: one arrival per dequantising warp
  uint64_t tfull[2], tempty[2], mma_done;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kQSmemBytes =
    1024 + QSTAGES * (QA_BYTES + QB_BYTES) + QW_STAGES * QW_BYTES + sizeof(QTail);
static_assert(kQSmemBytes <= 232448, "shared memory per CTA");

// MN-major B with 128-byte swizzling: 64 outputs (128 B) per input-channel row,
// 8-row core groups 1024 B apart (SBO), 64-output boxes QB_BOX apart (LBO).
__device__ __forceinline__ uint64_t desc_b_mn(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((QB_BOX >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

__device__ __forceinline__ void q_tile_coords(int tile, int num_m, int num_n, int &m_blk, int &n_blk) {
  const int per_group = QGROUP_M * num_n;
  const int g = tile / per_group;
  const int first_m = g * QGROUP_M;
  const int gm = min(QGROUP_M, num_m - first_m);
  const int local = tile - g * per_group;
  m_blk = first_m + local % gm;
  n_blk = local / gm;
}

// Split-K: tile = (output tile, K split), split fastest; split sp of S covers
// K steps [sp num_kb / S, (sp + 1) num_kb / S).
__device__ __forceinline__ void q_tile_split(int tile, int num_m, int num_n, int splits, int num_kb,
                                             int &m_blk, int &n_blk, int &sp, int &kb0, int &kb1) {
  sp = tile % splits;
  q_tile_coords(tile / splits, num_m, num_n, m_blk, n_blk);
  kb0 = (int)((int64_t)sp * num_kb / splits);
  kb1 = (int)((int64_t)(sp + 1) * num_kb / splits);
}

// fp16 pairs {1024 + nibble p, 1024 + nibble p + 4}, p = 0..3, of a word
__device__ __forceinline__ void nib_pairs(uint32_t w, __half2 (&h)[4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t bits = ((w >> (4 * p)) & 0x000F000Fu) | 0x64006400u;
    h[p] = *reinterpret_cast<const __half2 *>(&bits);
  }
}

// scales of outputs (p, p + 4), p = 0..3, from 8 consecutive fp16 scales
__device__ __forceinline__ void scale_pairs(uint4 sc, __half2 (&h)[4]) {
  const uint32_t lo[2] = {sc.x, sc.y}, hi[2] = {sc.z, sc.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    // half p of the first four, half p of the last four
    const uint32_t a = lo[p >> 1], b = hi[p >> 1];
    const uint32_t bits = __byte_perm(a, b, (p & 1) ? 0x7632u : 0x5410u);
    h[p] = *reinterpret_cast<const __half2 *>(&bits);
  }
}

// 8 weights RN16((q - z) * scale) of one word in the order 0,4,1,5,2,6,3,7;
// (1024 + q) - (1024 + z) is exact
__device__ __forceinline__ uint4 dequant_word(uint32_t w, const __half2 (&zp)[4], const __half2 (&sp)[4]) {
  __half2 qp[4];
  nib_pairs(w, qp);
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const __half2 r = __hmul2(__hsub2(qp[p], zp[p]), sp[p]);
    o[p] = *reinterpret_cast<const uint32_t *>(&r);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void q_abort(QTail *t, DevStatus *st, uint32_t where) {
  dev_fail(st, kDevTimeout, where);
  *reinterpret_cast<volatile int *>(&t->abort_flag) = 1;
}
}  // namespace

__global__ void __launch_bounds__(Q_THREADS, 1) w4a16_gemm_kernel(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
    const int32_t *__restrict__ qzeros, const __half *__restrict__ scales, int64_t T, int64_t out,
    int group, int num_m, int num_n, int num_kb, int splits, __half *__restrict__ Y, int64_t ldy,
    float *__restrict__ partials, DevStatus *st, uint32_t max_polls) {
  extern __shared__ uint8_t q_smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(q_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + QSTAGES * QA_BYTES;
  uint8_t *sW = sB + QSTAGES * QB_BYTES;
  QTail *tail = reinterpret_cast<QTail *>(sW + QW_STAGES * QW_BYTES);
  volatile int *abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = num_m * num_n * splits;
  const int64_t words = out / 8;  // int32 words per qweight / qzeros row

  if (threadIdx.x == 0) {
    for (int s = 0; s < QSTAGES; ++s) {
      mbar_init(&tail->ld[s], 1);
      mbar_init(&tail->full[s], QN_DEQ);
      mbar_init(&tail->empty[s], 1);
    }
    for (int s = 0; s < QW_STAGES; ++s) {
      mbar_init(&tail->wld[s], 1);
      mbar_init(&tail->wempty[s], QN_DEQ);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tail->tfull[a], 1);
      mbar_init(&tail->tempty[a], 4);
    }
    mbar_init(&tail->mma_done, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmX);
  if (warp == QW_WPROD && lane == 0) tma_prefetch_desc(&tmW);
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, QTMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ X by TMA
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int m_blk, n_blk, sp, kb0, kb1;
        q_tile_split(tile, num_m, num_n, splits, num_kb, m_blk, n_blk, sp, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_long(&tail->empty[stage], phase ^ 1u, max_polls, abort_flag)) {
            q_abort(tail, st, 0xD00u + stage);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tail->ld[stage], QA_BYTES);
          tma_load_2d(sA + stage * QA_BYTES, &tmX, &tail->ld[stage], kb * QBK, m_blk * QBM);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == QSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok || *abort_flag)
        for (int s = 0; s < QSTAGES; ++s)
          if (issued & (1u << s))
            (void)mbar_wait_bounded(&tail->ld[s], (issued_parity >> s) & 1u, Q_DRAIN, nullptr);
    }
  } else if (warp == QW_WPROD) {
    // ------------------------------------------------------------ packed words by TMA
    // Their own ring: a slot is refilled as soon as the dequantising warps have
    // read it, so the words of a step land long before its B slot frees.
    if (lane == 0) {
      int ws = 0;
      uint32_t wphase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int m_blk, n_blk, sp, kb0, kb1;
        q_tile_split(tile, num_m, num_n, splits, num_kb, m_blk, n_blk, sp, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_long(&tail->wempty[ws], wphase ^ 1u, max_polls, abort_flag)) {
            q_abort(tail, st, 0xD50u + ws);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tail->wld[ws], QW_BYTES);
          tma_load_2d(sW + ws * QW_BYTES, &tmW, &tail->wld[ws], n_blk * (QBN / 8), kb * QBK);
          issued |= 1u << ws;
          issued_parity = (issued_parity & ~(1u << ws)) | (wphase << ws);
          if (++ws == QW_STAGES) {
            ws = 0;
            wphase ^= 1u;
          }
        }
      }
      if (!ok || *abort_flag)
        for (int s = 0; s < QW_STAGES; ++s)
          if (issued & (1u << s))
            (void)mbar_wait_bounded(&tail->wld[s], (issued_parity >> s) & 1u, Q_DRAIN, nullptr);
    }
  } else if (warp >= QW_DEQ) {
    // ------------------------------------------------------------ dequantise W
    const int dt = threadIdx.x - QW_DEQ * 32;  // 0..255
    const int col = dt & 31;                   // word column: outputs 8 col .. 8 col + 7
    const int row0 = dt >> 5;                  // input-channel rows row0 + QN_DEQ i
    // (QN_DEQ is a multiple of 8, so every row of this thread has k & 7 = row0 & 7)
    const uint32_t chunk_off = (uint32_t)(col >> 3) * QB_BOX + (uint32_t)row0 * 128u +
                               ((uint32_t)((col & 7) ^ (row0 & 7)) << 4);
    int stage = 0, ws = 0;
    uint32_t phase = 0, wphase = 0;
    // the (tile, K step) sequence of this CTA, one step ahead for the word loads
    int tile = blockIdx.x, kb = 0, kb_end = 0;
    // this thread's qweight column in tile tl, and the tile's K steps
    auto word_col = [&](int tl, int &k0, int &k1) {
      int m_blk, n_blk, sp;
      q_tile_split(tl, num_m, num_n, splits, num_kb, m_blk, n_blk, sp, k0, k1);
      return (int64_t)n_blk * (QBN / 8) + col;
    };
    // zero words and scales of one K step: rows 0..31 of the step use group
    // h = 0, rows 32..63 group h = 1 (the same group unless g = 32); loaded one
    // step ahead (the packed words themselves arrive by TMA with the X tile)
    uint32_t znext[2];
    uint4 snext[2];
    auto load_zs = [&](int64_t wc, int k_blk) {
      const bool ok_c = wc < words;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t gi = ((int64_t)k_blk * QBK + 32 * h) / group;
        znext[h] = ok_c ? (uint32_t)__ldg(qzeros + gi * words + wc) : 0u;
        snext[h] = ok_c ? __ldg(reinterpret_cast<const uint4 *>(scales + gi * out + 8 * wc))
                        : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    int64_t wcol = tile < num_tiles ? word_col(tile, kb, kb_end) : 0;
    if (tile < num_tiles) load_zs(wcol, kb);
    bool ok = true;
    while (ok && tile < num_tiles) {
      uint32_t zw[2];
      uint4 sc[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        zw[h] = znext[h];
        sc[h] = snext[h];
      }
      int ntile = tile, nkb = kb + 1, nkb_end = kb_end;
      int64_t nwcol = wcol;
      if (nkb == kb_end) {
        ntile += gridDim.x;
        nwcol = ntile < num_tiles ? word_col(ntile, nkb, nkb_end) : 0;
      }
      if (ntile < num_tiles) load_zs(nwcol, nkb);
      __half2 zp[2][4], sp[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        nib_pairs(zw[h], zp[h]);
        scale_pairs(sc[h], sp[h]);
      }
      // the step's packed words have landed, and the MMAs that last read this
      // B slot are done
      int got = 1;
      if (lane == 0)
        got = mbar_wait_long(&tail->wld[ws], wphase, max_polls, abort_flag) &&
              mbar_wait_long(&tail->empty[stage], phase ^ 1u, max_polls, abort_flag);
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) {
        if (lane == 0) q_abort(tail, st, 0xD10u + stage);
        ok = false;
        break;
      }
      // words past `out` were filled with zeros by TMA; their zeros and scales
      // are zero too, so they give 0
      const uint32_t *wsrc = reinterpret_cast<const uint32_t *>(sW + ws * QW_BYTES) + row0 * 32 + col;
      uint8_t *bst = sB + stage * QB_BYTES + chunk_off;
      // all eight words first: the B stores below may not be reordered above
      // loads the compiler cannot prove disjoint, so loads come first explicitly
      uint32_t wv[Q_WORDS];
#pragma unroll
      for (int i = 0; i < Q_WORDS; ++i) wv[i] = wsrc[i * QN_DEQ * 32];
#pragma unroll
      for (int i = 0; i < Q_WORDS; ++i) {
        // row row0 + QN_DEQ i lies in 0..31 (zero and scale group h = 0) for the
        // first half of i and in 32..63 (h = 1) for the second
        constexpr int kHalf = Q_WORDS / 2;
        const uint4 v = dequant_word(wv[i], zp[i < kHalf ? 0 : 1], sp[i < kHalf ? 0 : 1]);
        *reinterpret_cast<uint4 *>(bst + i * QN_DEQ * 128) = v;  // row row0 + QN_DEQ i, same swizzle
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tail->wempty[ws]);  // every word of the slot was used above
        mbar_arrive(&tail->full[stage]);
      }
      if (++stage == QSTAGES) {
        stage = 0;
        phase ^= 1u;
      }
      if (++ws == QW_STAGES) {
        ws = 0;
        wphase ^= 1u;
      }
      tile = ntile;
      kb = nkb;
      kb_end = nkb_end;
      wcol = nwcol;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued_any = false;
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = 0;  // one tile in TMEM: columns 0..255 rows 0..127, 256..511 rows 128..255
        const uint32_t acc_phase = it & 1;
        if (!mbar_wait_long(&tail->tempty[acc], acc_phase ^ 1u, max_polls, abort_flag)) {
          q_abort(tail, st, 0xD20u + acc);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base;
        int m_blk, n_blk, sp, kb0, kb1;
        q_tile_split(tile, num_m, num_n, splits, num_kb, m_blk, n_blk, sp, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_long(&tail->full[stage], phase, max_polls, abort_flag) ||
              !mbar_wait_bounded(&tail->ld[stage], phase, max_polls, abort_flag)) {  // X tile
            q_abort(tail, st, 0xD30u + stage);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * QA_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * QB_BYTES);
#pragma unroll
          for (int k = 0; k < QBK / 16; ++k) {
            const uint64_t bd = desc_b_mn(b_addr + k * 2048);
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tc_mma_f16(d_tmem + h * QBN, smem_desc_k_sw128(a_addr + h * QA_HALF + k * 32), bd, IDESC_Q,
                         (kb != kb0 || k != 0) ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(&tail->empty[stage]);
          if (++stage == QSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tail->tfull[acc]);
      }
      if (issued_any) {
        tc_commit(&tail->mma_done);
        (void)mbar_wait_bounded(&tail->mma_done, 0, Q_DRAIN, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int acc = 0;
      const uint32_t acc_phase = it & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait_long(&tail->tfull[acc], acc_phase, max_polls, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) q_abort(tail, st, 0xD40u + acc);
        break;
      }
      tc_fence_after();
      int m_blk, n_blk, sp, kb0, kb1;
      q_tile_split(tile, num_m, num_n, splits, num_kb, m_blk, n_blk, sp, kb0, kb1);
#pragma unroll 1
      for (int c2 = 0; c2 < 2 * QBN; c2 += 32) {
        const int h = c2 / QBN, c = c2 % QBN;  // accumulator half (rows 128 h ..) and column
        const int64_t t_row = (int64_t)m_blk * QBM + h * QMM + q * 32 + lane;
        float v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c2, v);
        tmem_ld_wait();
        const int64_t o0 = (int64_t)n_blk * QBN + c;
        if (partials && t_row < T && AWQ_IN_BOUNDS(sp < splits, 0xB060u)) {
          // split-K: this split's fp32 sums, in output order, for the reduction
          float *prow = partials + ((int64_t)sp * T + t_row) * out + o0;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (o0 + 8 * u >= out) break;  // out % 8 == 0
            // accumulator column 8u + 2p holds output 8u + p, column 8u + 2p + 1 output 8u + p + 4
            const float4 lo = make_float4(v[8 * u + 0], v[8 * u + 2], v[8 * u + 4], v[8 * u + 6]);
            const float4 hi = make_float4(v[8 * u + 1], v[8 * u + 3], v[8 * u + 5], v[8 * u + 7]);
            *reinterpret_cast<float4 *>(prow + 8 * u) = lo;
            *reinterpret_cast<float4 *>(prow + 8 * u + 4) = hi;
          }
        } else if (t_row < T) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (o0 + 8 * u >= out) break;  // out % 8 == 0
            // accumulator column 8u + 2p holds output 8u + p, column 8u + 2p + 1 output 8u + p + 4
            uint32_t hw[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const int e0 = 2 * h, e1 = 2 * h + 1;  // outputs of this half2
              const int c0 = e0 < 4 ? 2 * e0 : 2 * (e0 - 4) + 1, c1 = e1 < 4 ? 2 * e1 : 2 * (e1 - 4) + 1;
              const __half2 hv = __floats2half2_rn(v[8 * u + c0], v[8 * u + c1]);
              hw[h] = *reinterpret_cast<const uint32_t *>(&hv);
            }
            *reinterpret_cast<uint4 *>(Y + t_row * ldy + o0 + 8 * u) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, QTMEM_COLS);
  }
}

// The dequantised weights Wd [out, in] fp16, Wd[o][j] = RN16((q - z) scale) --
// the values the GEMM above builds tile by tile -- written once for a product
// with many tokens.  A block turns a 128-input x 64-output tile of packed
// words (input-major) into output-major rows through shared memory, so both
// the word loads and the 16-byte row stores are contiguous.
__global__ void __launch_bounds__(256) w4a16_dequant_kernel(
    const int32_t *__restrict__ qweight, const int32_t *__restrict__ qzeros,
    const __half *__restrict__ scales, int64_t in, int64_t out, int group, __half *__restrict__ Wd) {
  constexpr int TJ = 128, TO = 64, WPR = TO / 8;  // inputs, outputs, words per input row
  // [output][input] with the 16-byte chunks of row r XOR-swizzled by r / 8, so
  // that the 2-byte writes of one warp (8 word columns, i.e. rows 8 apart)
  // fall in different banks and the 16-byte row reads stay aligned
  __shared__ __align__(16) __half tile[TO][TJ];
  // outputs along x (up to 2^22 / 64 blocks), inputs along y (at most 2^20 / 128)
  const int64_t o0 = (int64_t)blockIdx.x * TO, j0 = (int64_t)blockIdx.y * TJ;
  const int64_t words = out / 8;
  // a thread converts the words of two consecutive input rows of one word
  // column (one group: group % 32 == 0) and writes each output's two weights
  // as one half2
#pragma unroll
  for (int i = 0; i < TJ * WPR / 512; ++i) {
    const int w = threadIdx.x + 256 * i;
    const int jp = w / WPR, ow = w % WPR;  // input row pair of the tile, word column
    const int jj = 2 * jp;
    const int64_t j = j0 + jj, wc = o0 / 8 + ow;
    uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
    if (j < in && wc < words) {  // in % 64 == 0: rows j and j + 1 are both in
      const int64_t gi = j / group;
      __half2 zp[4], sp[4];
      nib_pairs((uint32_t)__ldg(qzeros + gi * words + wc), zp);
      scale_pairs(__ldg(reinterpret_cast<const uint4 *>(scales + gi * out + 8 * wc)), sp);
      const int32_t *qp = qweight + j * words + wc;
      v0 = dequant_word((uint32_t)__ldg(qp), zp, sp);
      v1 = dequant_word((uint32_t)__ldg(qp + words), zp, sp);
    }
    // v0 / v1 hold outputs 0,4,1,5,2,6,3,7 of the word in rows jj / jj + 1
    const uint32_t h0[4] = {v0.x, v0.y, v0.z, v0.w}, h1[4] = {v1.x, v1.y, v1.z, v1.w};
    const int col = (((jj >> 3) ^ ow) << 3) | (jj & 7);  // rows 8 ow .. 8 ow + 7 share the swizzle
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      // output p: low halves of row jj and row jj + 1; output p + 4: the high halves
      const uint32_t lo = __byte_perm(h0[p], h1[p], 0x5410u), hi = __byte_perm(h0[p], h1[p], 0x7632u);
      *reinterpret_cast<uint32_t *>(&tile[8 * ow + p][col]) = lo;
      *reinterpret_cast<uint32_t *>(&tile[8 * ow + p + 4][col]) = hi;
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < TO * (TJ / 8) / 256; ++i) {
    const int c = threadIdx.x + 256 * i;
    const int oo = c / (TJ / 8), jc = c % (TJ / 8);  // output row, 8-input chunk
    const int64_t o = o0 + oo, j = j0 + 8 * jc;
    if (o < out && j < in)  // in % 64 == 0: a chunk is whole
      *reinterpret_cast<uint4 *>(Wd + o * in + j) =
          *reinterpret_cast<const uint4 *>(&tile[oo][8 * (jc ^ (oo >> 3))]);
  }
}

cudaError_t launch_w4a16_dequant(const int32_t *qweight, const int32_t *qzeros, const __half *scales,
                                 int64_t in, int64_t out, int group, __half *Wd, cudaStream_t stream) {
  if (in % 64 != 0 || out % 8 != 0 || group % 32 != 0) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((out + 63) / 64), (unsigned)((in + 127) / 128));
  w4a16_dequant_kernel<<<grid, 256, 0, stream>>>(qweight, qzeros, scales, in, out, group, Wd);
  return cudaGetLastError();
}

// Y[t][o] = RN16(sum over splits s of partials[s][t][o]), the splits added in
// order (a fixed summation order: the result does not depend on scheduling).
__global__ void w4a16_splitk_reduce_kernel(const float *__restrict__ partials, int splits, int64_t T,
                                           int64_t out, __half *__restrict__ Y, int64_t ldy) {
  const int64_t n4 = T * out / 4;  // out % 8 == 0
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = __ldcs(reinterpret_cast<const float4 *>(partials) + i);
    for (int sp = 1; sp < splits; ++sp) {
      const float4 v = __ldcs(reinterpret_cast<const float4 *>(partials + (int64_t)sp * T * out) + i);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    const int64_t e = 4 * i, t = e / out, o = e - t * out;
    const __half2 a = __floats2half2_rn(acc.x, acc.y), b = __floats2half2_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t *>(&a);
    pk.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(Y + t * ldy + o) = pk;
  }
}

// ---------------------------------------------------------------------------
// Decode: up to kGemvMaxT tokens.  The product reads each packed word once and
// does T x 8 multiply-adds with it, so it is bound by reading the weights, not
// by the tensor cores: a CUDA-core kernel streams the words instead.  The
// matrix is only a few MB, so the design goal is to have nearly all of it in
// flight at once: a block covers 256 outputs (a warp's 32 lanes read 32
// consecutive words of an input row: 128 contiguous bytes) and 256 input rows
// (one K split), warp w rows 32w..32w+31 (inside one group: group | 32), and a
// lane issues the loads of 32 / 16 / 8 of its rows together (T <= 2 / 4 / 8,
// as registers allow).  The block's X[t][j] are staged in shared memory as
// fp32 pairs (x, x); a lane dequantises each word to the fp16 weights
// RN16((q - z) scale) (the values the GEMM forms use), whose halves pair
// outputs (p, p + 4), widens them and accumulates with packed f32x2 FMAs, rows
// in ascending order.  The warps' sums are added in a fixed order through
// shared memory; with several K splits (blocks along y) each writes fp32 sums
// for the split-K reduction, else the block rounds Y itself.
// ---------------------------------------------------------------------------
constexpr int kGemvMaxT = 8;
constexpr int kGemvOut = 256;   // outputs per block
constexpr int kGemvWarps = 8;

// rows per warp; a K split is 8 warps x that (256 rows): about two blocks
// per SM for a 4096 x 4096 layer, and partial sums of 1/32 of the weights'
// bytes per token
__host__ __device__ constexpr int gemv_warp_rows(int) { return 32; }

template <int TT>
__global__ void __launch_bounds__(kGemvWarps * 32, 2) w4a16_gemv_kernel(
    const __half *__restrict__ X, int64_t in, int64_t ldx, const int32_t *__restrict__ qweight,
    const int32_t *__restrict__ qzeros, const __half *__restrict__ scales, int64_t out, int group,
    int64_t k_per_split, __half *__restrict__ Y, int64_t ldy, float *__restrict__ partials) {
  constexpr int WR = gemv_warp_rows(TT);  // rows per warp and chunk
  constexpr int CH = kGemvWarps * WR;     // rows per chunk
  constexpr int RB = TT <= 2 ? 32 : TT <= 4 ? 16 : 8;  // rows whose words are loaded together
  constexpr int kRedT = TT < 4 ? TT : 4;  // tokens reduced per pass through shared memory
  constexpr int kXsBytes = CH * TT * 8;
  constexpr int kRedBytes = kGemvWarps * kRedT * (kGemvOut + 4) * 4;
  __shared__ __align__(16) unsigned char smem[kXsBytes > kRedBytes ? kXsBytes : kRedBytes];
  float2(*xs)[TT] = reinterpret_cast<float2(*)[TT]>(smem);  // [chunk row][token]: (x, x)
  float(*red)[kRedT][kGemvOut + 4] = reinterpret_cast<float(*)[kRedT][kGemvOut + 4]>(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t words = out / 8;
  const int64_t wc = (int64_t)blockIdx.x * (kGemvOut / 8) + lane;  // this lane's word column
  const bool col_ok = wc < words;
  const int64_t j0 = (int64_t)blockIdx.y * k_per_split;
  const int64_t j1 = j0 + k_per_split < in ? j0 + k_per_split : in;  // multiples of 64
  float2 acc[TT][4];  // outputs (p, p + 4) of the word, p = 0..3
#pragma unroll
  for (int t = 0; t < TT; ++t)
#pragma unroll
    for (int p = 0; p < 4; ++p) acc[t][p] = make_float2(0.0f, 0.0f);
  for (int64_t jc = j0; jc < j1; jc += CH) {
    const int rows = (int)(j1 - jc < CH ? j1 - jc : CH);  // a multiple of 64 or CH
    const int64_t jw = jc + WR * warp;
    const bool live = col_ok && WR * warp < rows;
    if (jc != j0) __syncthreads();  // the previous chunk's X is no longer read
    for (int i = threadIdx.x; i < rows * TT; i += kGemvWarps * 32) {
      const int t = i / rows, r = i - t * rows;
      const float x = AWQ_IN_BOUNDS(jc + r < in, 0xB061u) ? __half2float(__ldg(X + t * ldx + jc + r)) : 0.0f;
      xs[r][t] = make_float2(x, x);
    }
    __syncthreads();
    if (live) {
      const int64_t gi = jw / group;
      __half2 zp[4], sp[4];
      nib_pairs((uint32_t)__ldg(qzeros + gi * words + wc), zp);
      scale_pairs(__ldg(reinterpret_cast<const uint4 *>(scales + gi * out + 8 * wc)), sp);
#pragma unroll
      for (int rb = 0; rb < WR; rb += RB) {
        uint32_t wv[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r)
          wv[r] = AWQ_IN_BOUNDS(jw + rb + r < in, 0xB062u) ? (uint32_t)__ldg(qweight + (jw + rb + r) * words + wc)
                                                           : 0u;
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          const uint4 v = dequant_word(wv[r], zp, sp);
          const uint32_t hv[4] = {v.x, v.y, v.z, v.w};
          float2 wf[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) wf[p] = __half22float2(*reinterpret_cast<const __half2 *>(&hv[p]));
          const float2 *xr = xs[WR * warp + rb + r];
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            const float2 xx = xr[t];
#pragma unroll
            for (int p = 0; p < 4; ++p) acc[t][p] = __ffma2_rn(xx, wf[p], acc[t][p]);
          }
        }
      }
    }
  }
  __syncthreads();  // xs and red share the buffer
  // the warps' sums, added in a fixed order, kRedT tokens at a time
#pragma unroll
  for (int t0 = 0; t0 < TT; t0 += kRedT) {
#pragma unroll
    for (int t = 0; t < kRedT; ++t)
      if (t0 + t < TT) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          red[warp][t][8 * lane + p] = acc[t0 + t][p].x;
          red[warp][t][8 * lane + p + 4] = acc[t0 + t][p].y;
        }
      }
    __syncthreads();
    const int nt = TT - t0 < kRedT ? TT - t0 : kRedT;
    for (int i = threadIdx.x; i < nt * kGemvOut; i += blockDim.x) {
      const int t = i / kGemvOut, oo = i % kGemvOut;
      const int64_t o = (int64_t)blockIdx.x * kGemvOut + oo;
      if (o >= out) continue;
      float sum = red[0][t][oo];
#pragma unroll
      for (int w = 1; w < kGemvWarps; ++w) sum += red[w][t][oo];
      if (partials)
        partials[((int64_t)blockIdx.y * TT + t0 + t) * out + o] = sum;  // blockIdx.y < splits (the grid)
      else
        Y[(t0 + t) * ldy + o] = __float2half_rn(sum);
    }
    __syncthreads();
  }
}

// one K split per 8 x gemv_warp_rows(T) input rows
int w4a16_gemv_splits(int64_t T, int64_t in, int64_t out, int num_sms) {
  (void)out;
  (void)num_sms;
  if (T < 1 || T > kGemvMaxT) return 0;
  const int64_t ch = kGemvWarps * gemv_warp_rows((int)T);
  return (int)((in + ch - 1) / ch);
}

cudaError_t launch_w4a16_gemv(const __half *X, int64_t T, int64_t in, int64_t ldx,
                              const int32_t *qweight, const int32_t *qzeros, const __half *scales,
                              int64_t out, int group, __half *Y, int64_t ldy, float *partials,
                              int num_sms, cudaStream_t stream) {
  if (T < 1 || T > kGemvMaxT || in % 64 != 0 || out % 8 != 0 ||
      group % 32 != 0 || ldx % 8 != 0)
    return cudaErrorInvalidValue;
  // without room for partial sums, one block column covers all of `in`
  (void)num_sms;
  const int64_t k = partials ? kGemvWarps * gemv_warp_rows((int)T) : in;
  const int splits = (int)((in + k - 1) / k);
  float *part = splits > 1 ? partials : nullptr;
  dim3 grid((unsigned)((out + kGemvOut - 1) / kGemvOut), (unsigned)splits);
  const unsigned nt = kGemvWarps * 32;
  switch (T) {
    case 1: w4a16_gemv_kernel<1><<<grid, nt, 0, stream>>>(X, in, ldx, qweight, qzeros, scales, out, group, k, Y, ldy, part); break;
    case 2: w4a16_gemv_kernel<2><<<grid, nt, 0, stream>>>(X, in, ldx, qweight, qzeros, scales, out, group, k, Y, ldy, part); break;
    case 3: w4a16_gemv_kernel<3><<<grid, nt, 0, stream>>>(X, in, ldx, qweight, qzeros, scales, out, group, k, Y, ldy, part); break;
    case 4: w4a16_gemv_kernel<4><<<grid, nt, 0, stream>>>(X, in, ldx, qweight, qzeros, scales, out, group, k, Y, ldy, part); break;
    case 5: w4a16_gemv_kernel<5><<<grid, nt, 0, stream>>>(X, in, ldx, qweight, qzeros, scales, out, group, k, Y, ldy, part); break;
    case 6: w4a16_gemv_kernel<6><<<grid, nt, 0, stream>>>(X, in, ldx, qweight, qzeros, scales, out, group, k, Y, ldy, part); break;
    case 7: w4a16_gemv_kernel<7><<<grid, nt, 0, stream>>>(X, in, ldx, qweight, qzeros, scales, out, group, k, Y, ldy, part); break;
    default: w4a16_gemv_kernel<8><<<grid, nt, 0, stream>>>(X, in, ldx, qweight, qzeros, scales, out, group, k, Y, ldy, part); break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  const int64_t n4 = T * out / 4;
  w4a16_splitk_reduce_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, stream>>>(partials, splits, T, out,
                                                                              Y, ldy);
  return cudaGetLastError();
}

int w4a16_splits(int64_t T, int64_t in, int64_t out, int num_sms) {
  const int64_t tiles = ((T + QBM - 1) / QBM) * ((out + QBN - 1) / QBN);
  const int64_t num_kb = in / QBK;
  if (tiles * 2 > num_sms || num_kb < 8) return 1;
  // enough splits to fill the SMs, each with at least 4 K steps
  int64_t s = num_sms / tiles;
  if (s > num_kb / 4) s = num_kb / 4;
  return (int)(s < 1 ? 1 : s);
}

cudaError_t launch_w4a16_gemm(const __half *X, int64_t T, int64_t in, int64_t ldx,
                              const int32_t *qweight, const int32_t *qzeros, const __half *scales,
                              int64_t out, int group, __half *Y, int64_t ldy, float *partials,
                              int splits, DevStatus *st, uint32_t max_polls, int num_sms,
                              cudaStream_t stream) {
  if (in % QBK != 0 || out % 32 != 0 || group % 32 != 0) return cudaErrorInvalidValue;
  if (splits < 1 || splits > in / QBK || (splits > 1 && !partials)) return cudaErrorInvalidValue;
  CUtensorMap tmX, tmW;
  cudaError_t e = make_tmap_f16_box(&tmX, X, T, in, ldx, QBK, QBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_i32_box(&tmW, qweight, in, out / 8, out / 8, QBN / 8, QBK);  // words past out/8 read 0
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(w4a16_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kQSmemBytes);
  if (e != cudaSuccess) return e;
  const int num_m = (int)((T + QBM - 1) / QBM);
  const int num_n = (int)((out + QBN - 1) / QBN);
  const int tiles = num_m * num_n * splits;
  const int grid = tiles < num_sms ? tiles : num_sms;
  w4a16_gemm_kernel<<<grid, Q_THREADS, kQSmemBytes, stream>>>(
      tmX, tmW, qzeros, scales, T, out, group, num_m, num_n, (int)(in / QBK), splits, Y, ldy,
      splits > 1 ? partials : nullptr, st, max_polls);
  e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  const int64_t n4 = T * out / 4;
  const int64_t blocks = i64min((int64_t)num_sms * 8, (n4 + 255) / 256);
  w4a16_splitk_reduce_kernel<<<(unsigned)(blocks < 1 ? 1 : blocks), 256, 0, stream>>>(
      partials, splits, T, out, Y, ldy);
  return cudaGetLastError();
}

AWQ_BOUNDS_READER(bounds_status_w4a16)

}  // namespace awq
