// scorer.cu — the analytic tactic scorer: estimated time of a configuration,
// used to rank candidates without running them.
//
// FlashInfer PR 3948 ("perf(gemm): update mm_fp4 cute-dsl tactic heuristic and
// autotune over a top-N ranked list") replaces exhaustive tactic search with a
// heuristic that ranks tactics from the shape (wave quantisation, efficiency,
// feasibility) and tunes only the top N.  Here the ranking model is written
// from how this kernel spends its time, with its constants fitted (least
// squares on log time, per-shape offsets) to the tuner's measurements of
// every candidate on one B200 (precision_quantized_gemm_b200/fit_scorer.py,
// data in tables/b200_candidates.txt).  For one launch of configuration c:
//
//   rate   = min(in-flight bytes / L, per-SM bandwidth / CTAs per SM)
//            in-flight bytes = min(stages, K tiles of the slice) x stage bytes
//            (Little's law: a CTA keeps its ring's requests outstanding)
//   stream = bytes one CTA loads / rate
//   mma    = K tiles of the slice x (a0 + a1 tile_n [+ Block_FP8 promotion
//            a2 x columns one thread promotes + a3]) cycles / clock
//   body   = max(weight bytes / HBM bandwidth, waves x max(stream, mma))
//   epi    = e0 x pushed token columns / 16
//          + split-K: cluster: waves x (e1 + exchanged bytes / e2),
//                     second pass: e3, last CTA: e4,
//                     workspace modes: + 2 x split x M x N x 4 bytes / e5
//   time   = body + epi   (+ a per-shape constant that ranking ignores)
//
// Waves and CTAs per SM follow the launch's shared memory, register budget
// and TMEM columns.  On the 218 tuned shapes (34870 candidates) the
// top-ranked configuration is within 1.071x of the measured best (geomean),
// the best of the top 8 within 1.009x and of the top 16 within 1.003x (the
// fixed rule it replaced was 1.32x on an earlier 170-shape set).
#include <algorithm>
#include <cmath>
#include <vector>

#include "../../include/qgemm.h"
#include "internal.h"

namespace {

// Fitted constants (B200, 1965 MHz boost, measured HBM 6450.9 GB/s).
struct Model {
  double hbm_gbs = 6450.9;   // HBM bandwidth (measured copy bandwidth, held fixed)
  double lat_us = 1.38161;   // load latency under load seen by one CTA's ring
  double sm_gbs = 133.412;   // per-SM load bandwidth
  double a0 = 636.147, a1 = 0.873829;  // MMA-loop cycles per K tile: fixed, per tile_n column
  double a2 = 6.58675, a3 = 22.4012;   // Block_FP8 promotion cycles per K tile: per promoted column
  double clock_mhz = 1900.0;
  double e0 = 0.503163;      // epilogue per 16 pushed token columns, µs
  double e1 = 2.80164;       // cluster split-K exchange, fixed, µs per wave
  double e2 = 73.0506;       // cluster exchange bandwidth, GB/s per tile
  double e3 = 3.95830;       // second-pass launch, µs
  double e4 = 11.2845;       // last-CTA reduction, µs
  double e5 = 1180.85;       // workspace traffic bandwidth, GB/s
  // decode ("skinny") kernel: K-tile cycles of one compute warp, streaming
  // rate of one CTA (GB/s), fixed chain (µs)
  double s_tile = 300.0;
  double s_cta_gbs = 45.0;
  double s_chain = 2.3;
};
const Model kModel;

constexpr int kSmemPerSm = 233472;   // 228 KB of shared memory per SM

int tmem_columns(qg_format f, int tn) {
  int used;
  if (f == QG_BLOCK_FP8) used = (tn >= 256 ? 2 : 4) * tn;
  else if (f == QG_NVFP4) used = tn + 16 + 16 * (tn > 128 ? 2 : 1);
  else used = tn;
  int cols = 32;
  while (cols < used) cols *= 2;
  return cols;
}

int ctas_per_sm(qg_format f, int M, int K, const qg_config& c) {
  const bool blk = f == QG_BLOCK_FP8;
  const int regcap = (!blk && c.tile_n <= 64) ? 3 : ((!blk || c.tile_n <= 64) ? 2 : 1);
  const int tmemcap = 512 / tmem_columns(f, c.tile_n);
  const size_t smem = qg::config_smem(f, M, K, &c);
  const int smemcap = (int)(kSmemPerSm / (smem + 1024));
  return std::max(1, std::min(std::min(regcap, tmemcap), smemcap));
}

// The decode kernel: ceil(N / rows) x ceil(M / tile_n) CTAs, each streaming
// its rows (and tokens) over the whole of K through its ring; eight compute
// warps in K groups each take a share of the K tiles.  Calibrated on
// measured launches of this kernel (per-shape sweeps on one B200): a fixed
// chain of ~2.3 us (dependency release, activation tiles, the K-group sum,
// the stores), then the slice streaming at ~45 GB/s per CTA (shared when two
// CTAs sit on an SM), or the warps' MMA loop, whichever is longer, and never
// faster than the weights over HBM.
double estimate_skinny_us(qg_format f, int M, int N, int K, const qg_config& c, int sms) {
  const Model& m = kModel;
  const double rb = (double)K;
  const int kt = (int)((rb + 127) / 128);
  const double ctas = (double)((N + c.rows - 1) / c.rows) * ((M + c.tile_n - 1) / c.tile_n);
  const size_t smem = qg::config_smem(f, M, K, &c);
  const int cps = std::max(1, std::min(2, (int)(kSmemPerSm / (smem + 1024))));
  const double waves = std::ceil(ctas / ((double)sms * cps));
  const double cta_bytes = (double)(c.rows + c.tile_n) * 128.0 * kt;
  const double t_stream = cta_bytes / (m.s_cta_gbs * 1e3 / cps);
  const int kg = (c.tile_n == 8 ? 128 : 64) / c.rows;
  const double t_mma = std::ceil((double)kt / kg) * m.s_tile * std::max(1, c.tile_n / 16) / m.clock_mhz;
  const double body = std::max((double)N * rb / (m.hbm_gbs * 1e3), waves * std::max(t_stream, t_mma));
  return m.s_chain + body;
}

double estimate_us(qg_format f, int M, int N, int K, const qg_config& c, int sms) {
  if (c.variant == 1) return estimate_skinny_us(f, M, N, K, c, sms);
  if (c.variant == 3) {
    // CTA pairs (Block_FP8): the 256-wide tile kernel's estimate less the
    // promotion hand-off that the pair's 256-row MMAs halve per SM (a flat
    // 12 %; measured 10-27 % at 2048-16384 tokens; the tuner decides)
    qg_config t = c;
    t.variant = 0;
    t.tile_n = 256;
    t.stages = 3;
    return 0.88 * estimate_us(f, M, N, K, t, sms);
  }
  if (c.variant == 2) {
    // the persistent kernel: the tile kernel's estimate less the per-tile
    // set-up and epilogue that the next tile's MMAs hide (a flat 12 %; the
    // tuner's measurements decide).  Block_FP8's promotion epilogue runs on
    // the same SM as the next tile's MMAs and wins only at some shapes, so
    // there the tile kernel stays the untuned choice.
    // The base is the tile kernel at the persistent ring's own depth
    // (256-wide tiles, 4 stages; 3 for Block_FP8), not at c's: with one CTA
    // per SM the ring alone keeps the loads in flight, and the candidates
    // below are the rings deep enough for that (128-wide tiles a shade
    // behind 256-wide ones).
    qg_config t = c;
    t.variant = 0;
    t.tile_n = 256;
    t.stages = f == QG_BLOCK_FP8 ? 3 : 4;
    return (f == QG_BLOCK_FP8 ? 1.02 : 0.88) * (c.tile_n == 256 ? 1.0 : 1.03) * estimate_us(f, M, N, K, t, sms);
  }
  const Model& m = kModel;
  const double rb = f == QG_NVFP4 ? K / 2.0 : (double)K;
  const int kt = (int)((rb + 127) / 128);
  const int nkt = (kt + c.split_k - 1) / c.split_k;
  const int rows_p = c.swap_ab ? N : M, rows_q = c.swap_ab ? M : N;
  const double tiles = (double)((rows_p + 127) / 128) * ((rows_q + c.tile_n - 1) / c.tile_n);
  const double ctas = tiles * c.split_k;
  const int cps = ctas_per_sm(f, M, K, c);
  const double waves = std::ceil(ctas / ((double)sms * cps));
  const double stage_bytes = (128.0 + c.tile_n) * 128.0;
  const double inflight = std::min(c.stages, nkt) * stage_bytes;
  const double rate = std::min(inflight / m.lat_us, m.sm_gbs * 1e3 / cps);   // bytes per µs
  const double t_stream = (128.0 + c.tile_n) * nkt * 128.0 / rate;
  // Block_FP8 promotes on 4, 8 or 16 epilogue warps (tile_n < 128, 128,
  // 256): the columns one thread promotes per K tile set its cost
  const int pcols = c.tile_n / (c.tile_n >= 256 ? 4 : c.tile_n >= 128 ? 2 : 1);
  const double kcyc = m.a0 + m.a1 * c.tile_n + (f == QG_BLOCK_FP8 ? m.a2 * pcols + m.a3 : 0.0);
  const double t_mma = nkt * kcyc / m.clock_mhz;
  const double hbm_bytes = (double)N * rb + (M >= 1024 ? (double)M * rb : 0.0);
  const double body = std::max(hbm_bytes / (m.hbm_gbs * 1e3), waves * std::max(t_stream, t_mma));
  const double mt = c.swap_ab ? std::min(M, c.tile_n) : std::min(M, 128);
  const double pushed = c.swap_ab ? mt : c.tile_n;
  double epi = m.e0 * pushed / 16.0;
  if (c.split_k > 1) {
    if (c.reduce_mode == 0) {
      epi += waves * (m.e1 + c.split_k * 128.0 * pushed * 4.0 / (m.e2 * 1e3));
    } else {
      epi += (c.reduce_mode == 1 ? m.e3 : m.e4) + 2.0 * c.split_k * M * (double)N * 4.0 / (m.e5 * 1e3);
    }
  }
  return body + epi;
}

}  // namespace

namespace qg {
// The candidate grid: split_k over powers of two up to the K tiles (and 256),
// Swap-AB tiles no wider than twice the token count, standard tiles for at
// least 64 tokens, rings of 3, 4, 6 or 8 stages, every reduction mode.
void candidate_grid(qg_format f, int M, int N, int K, qg_config* out, int max_out, int* n_out) {
  (void)N;
  const int kt = (int)(((f == QG_NVFP4 ? K / 2 : K) + 127) / 128);
  const int tiles_swap[] = {16, 32, 64, 128, 256};
  const int tiles_std[] = {256, 128, 64};
  const int stage_opts[] = {3, 4, 6, 8};
  int n = 0;
  for (int swap = 0; swap <= 1; ++swap) {
    const int* tiles = swap ? tiles_swap : tiles_std;
    const int ntiles = swap ? 5 : 3;
    for (int ti = 0; ti < ntiles; ++ti) {
      const int tn = tiles[ti];
      if (swap && tn > 2 * std::max(16, M)) continue;     // tokens would mostly be padding
      if (!swap && (tn < 64 || M < 64)) continue;         // standard needs a real 128-token tile
      for (int sk = 1; sk <= 256 && sk <= kt; sk *= 2)
        for (int st : stage_opts)
          for (int rm = 0; rm <= (sk > 1 ? 2 : 0); ++rm) {
            if (n < max_out) {
              qg_config c = {};
              c.split_k = sk;
              c.swap_ab = swap;
              c.tile_n = tn;
              c.stages = st;
              c.reduce_mode = rm;
              out[n] = c;
            }
            ++n;
          }
    }
  }
  // the persistent kernel (8-bit formats, at least 256 tokens): the rings
  // that keep about 190 KB of operands in flight per SM (256-wide tiles with
  // 4 stages, 128-wide with 6; Block_FP8, whose partials and scales take the
  // rest of shared memory, 256-wide with 3).  Shallower rings measured up to
  // 1.6x slower at one CTA per SM.
  if (f != QG_NVFP4 && M >= 256) {
    const int rings[2][2] = {{256, f == QG_BLOCK_FP8 ? 3 : 4}, {128, 6}};
    for (int r = 0; r < (f == QG_BLOCK_FP8 ? 1 : 2); ++r) {
      if (n < max_out) {
        qg_config c = {};
        c.split_k = 1;
        c.swap_ab = 0;
        c.tile_n = rings[r][0];
        c.stages = rings[r][1];
        c.reduce_mode = 0;
        c.variant = 2;
        out[n] = c;
      }
      ++n;
    }
  }
  // CTA pairs (Block_FP8): 256 x 256 pair tiles with rings of 3, 4 or 6
  // stages, where there are pair tiles for most of the SM pairs (fewer lost
  // to the tile kernel with split-K: 28-40 tiles measured 4-80 % slower)
  const long long pair_tiles = (long long)((M + 255) / 256) * ((N + 255) / 256);
  if (f == QG_BLOCK_FP8 && pair_tiles >= 60) {
    for (int st : {3, 4, 6}) {
      if (n < max_out) {
        qg_config c = {};
        c.split_k = 1;
        c.swap_ab = 0;
        c.tile_n = 256;
        c.stages = st;
        c.reduce_mode = 0;
        c.variant = 3;
        out[n] = c;
      }
      ++n;
    }
  }
  // the decode kernel (8-bit formats, up to 32 tokens per CTA): rows per
  // CTA, and rings of 8, 16, 32 or every K tile (up to 64) rounded to the K
  // groups
  if (f != QG_NVFP4 && M <= 64) {
    const int rows_opts[] = {8, 16, 32, 64};
    const int ring_opts[] = {8, 16, 32, 64};
    for (int tm : {8, 16, 32}) {
      if ((tm == 32 && M <= 16) || (tm == 8 && M > 8)) continue;
      for (int r : rows_opts) {
        if (tm == 8 && r < 16) continue;
        const int kg = (tm == 8 ? 128 : 64) / r;
        int prev = 0;
        for (int ro : ring_opts) {
          int st = std::min(ro, ((kt + kg - 1) / kg) * kg);
          st = std::max(kg, (st / kg) * kg);
          if (st < 2) st = 2 * kg > 64 ? kg : 2 * kg;
          if (st == prev) continue;
          prev = st;
          if (n < max_out) {
            qg_config c = {};
            c.split_k = 1;
            c.swap_ab = 1;
            c.tile_n = tm;
            c.stages = st;
            c.reduce_mode = 0;
            c.variant = 1;
            c.rows = r;
            out[n] = c;
          }
          ++n;
        }
      }
    }
  }
  *n_out = n;
}
}  // namespace qg

extern "C" {

qg_status qgemm_score_config(qg_format f, int M, int N, int K, const qg_config* cfg, double* est_us) {
  if (!cfg || !est_us || (int)f < 0 || (int)f > 3 || M <= 0 || N <= 0 || K <= 0) return QG_ERR_INVALID_ARG;
  const qg_status s = qg::config_check(f, M, N, K, cfg);
  if (s != QG_OK) return s;
  *est_us = estimate_us(f, M, N, K, *cfg, qg::device_sm_count());
  return QG_OK;
}

qg_status qgemm_rank_configs(qg_format f, int M, int N, int K, qg_config* out, int max_out, double* est_us,
                             int* n_out) {
  if (!n_out || (max_out > 0 && !out) || max_out < 0 || (int)f < 0 || (int)f > 3 || M <= 0 || N <= 0 ||
      K <= 0)
    return QG_ERR_INVALID_ARG;
  int total = 0;
  qg::candidate_grid(f, M, N, K, nullptr, 0, &total);
  std::vector<qg_config> grid((size_t)total);
  qg::candidate_grid(f, M, N, K, grid.data(), total, &total);
  const int sms = qg::device_sm_count();
  std::vector<std::pair<double, int>> scored;
  for (int i = 0; i < total; ++i)
    if (qg::config_check(f, M, N, K, &grid[i]) == QG_OK)
      scored.emplace_back(estimate_us(f, M, N, K, grid[i], sms), i);
  // ties keep grid order, so the ranking is deterministic
  std::stable_sort(scored.begin(), scored.end(),
                   [](const std::pair<double, int>& a, const std::pair<double, int>& b) { return a.first < b.first; });
  const int n = std::min((int)scored.size(), max_out);
  for (int i = 0; i < n; ++i) {
    out[i] = grid[scored[i].second];
    if (est_us) est_us[i] = scored[i].first;
  }
  *n_out = n;
  return QG_OK;
}

}  // extern "C"
