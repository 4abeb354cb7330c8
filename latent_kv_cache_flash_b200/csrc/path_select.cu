// Runtime choice between the two decode paths.  The same weights serve both
// ("GQLA" chatpaper.ai Abstract: an MQA-absorb path and a GQA path over the
// same parameters, the runtime taking whichever suits the hardware; "GQLA"
// scholarbro.com Abstract: the choice follows the GPU's compute-to-bandwidth
// balance).  The estimate models this library's own kernels: which resource
// bounds each kernel, its tile shape and its measured efficiency against the
// copy bandwidth and the dense bf16 tensor rate of the GPU.
#include <math.h>

#include "launch.h"
#include "tc.h"

namespace gqla {

namespace {

// Copy bandwidth and dense bf16 tensor rate measured on a B200 (STREAM-style
// copy; cuBLAS bf16 GEMM burst): the defaults when no hardware is given.
constexpr double kDefaultHbmGbs = 6559.0;
constexpr double kDefaultTcTflops = 1656.2;

// Efficiencies of the kernels against those two rates, and their fixed
// costs, measured on a B200 over the crossover grid (n_h 128, G 1..128,
// s_q 1..4, B32, L 32K) and the DeepSeek-V3-shaped context sweep (B64,
// L 8K..64K):
constexpr double kEtaStream = 1.08;     // GQA mma.sync kernel, <= 16 rows a group: K/V read stream (1.07..1.10 of the copy rate)
constexpr double kEtaStreamWide = 1.0;  // the same kernel at 17..63 rows a group, where its MMAs slow each CTA's stream
constexpr double kEtaWideTc = 0.60;     // GQA tcgen05 kernel: a 128-row block-tile, full or not (softmax-bound)
constexpr double kEtaWideBw = 0.98;     // its K/V stream: a wave's first row blocks share HBM (the others hit L2)
constexpr double kWideCtaUs = 11.0;     // its CTA prologue (query into TMEM) + epilogue (merge of two states, output)
constexpr double kEtaAbsorbTc = 0.42;   // absorb tcgen05 kernel: M=64 tiles, N=64 score MMAs
constexpr double kEtaAbsorbBw = 0.90;   // a CTA's latent tile loads (every row block loads each tile into its SM)
constexpr double kLaunchUs = 3.0;       // one kernel launch on a busy stream
constexpr double kAbsorbCtaUs = 9.0;    // absorb CTA prologue (q~ into TMEM) + epilogue (64 x 512 fp32 out)
// The absorbed-query GEMM and the fused split merge + up-projection, beside
// reading the split partials back: latency-bound small launches, about 31 us
// together from 4K to 16K rows.
constexpr double kAbsorbSideUs = 31.0;

struct Rates {
  double bw_sm;   // bytes/us per SM
  double tc_sm;   // flop/us per SM
  double bw;      // bytes/us
  int sms;
};

// Split partials read back by the merge (their writes overlap the decode).
double combine_us(const Problem& p, int D, const Rates& r) {
  const double bytes = (double)p.plan.num_splits * (double)p.rows * (D + 1) * 4;
  return bytes / r.bw + kLaunchUs;
}

double absorb_us(const Problem& p, long long T, const Rates& r) {
  const auto& d = p.d;
  const int es = d.dtype == GQLA_F32 ? 4 : 2;
  const long long rb = (d.n_h * d.s_q + 63) / 64;
  const double tiles = (double)T / 64.0 + 0.5 * p.ly.batch;           // sum over sequences of ceil(L / 64)
  const double flops_tile = 2.0 * 64 * 64 * (2.0 * d.r + d.d_rope);   // QK over r + d_rope, PV over r
  const double bytes_tile = 64.0 * (d.r + d.d_rope) * es;
  const double t_tile = fmax(flops_tile / (r.tc_sm * kEtaAbsorbTc), bytes_tile / (r.bw_sm * kEtaAbsorbBw));
  // one CTA per SM: whole waves of CTAs, each its share of the tiles
  const double ctas = (double)p.ly.batch * p.plan.num_splits * rb;
  const double dec = ceil(ctas / r.sms) * (kAbsorbCtaUs + tiles * rb / ctas * t_tile);
  // absorbed-query GEMM + merge of the split partials and up-projection
  const double aux = kAbsorbSideUs + (double)p.plan.num_splits * (double)p.rows * (d.r + 1) * 4 / r.bw;
  return dec + aux;
}

double gqa_us(const Problem& p, long long T, const Rates& r) {
  const auto& d = p.d;
  const int es = d.dtype == GQLA_F32 ? 4 : 2;
  const double row_bytes = ((double)p.kr.pitch + (double)d.G * d.d_v) * es;   // K + V of one token, all groups
  const double tiles = (double)T / 64.0 + 0.5 * p.ly.batch;
  double dec;
  if (tc_gqa_wide_supports(p)) {
    // per wave: each CTA's tiles at the tensor rate, or at the wave's share
    // of HBM (only the first row block of a tile reads it from HBM)
    const long long rb = (p.m * d.s_q + 127) / 128;
    const double flops_tile = 2.0 * 128 * 64 * (p.d_qk + d.d_v);
    const double bytes_tile = 64.0 * row_bytes / d.G;
    const double t_tc = flops_tile / (r.tc_sm * kEtaWideTc);
    const double ctas = (double)p.ly.batch * d.G * p.plan.num_splits * rb;
    const double tiles_cta = tiles * d.G * rb / ctas;
    dec = 0.0;
    for (double left = ctas; left > 0.0; left -= r.sms) {
      const double w = fmin(left, (double)r.sms);
      const double t_hbm = w / rb * bytes_tile / (r.bw * kEtaWideBw);
      dec += kWideCtaUs + tiles_cta * fmax(t_tc, t_hbm);
    }
  } else {
    dec = (double)T * row_bytes / (r.bw * (p.m * d.s_q <= 16 ? kEtaStream : kEtaStreamWide));
  }
  return dec + kLaunchUs + (p.plan.num_splits > 1 ? combine_us(p, d.d_v, r) : 0.0);
}

}  // namespace

}  // namespace gqla

using namespace gqla;

extern "C" gqla_status gqla_select_path(const gqla_dims* dims, const gqla_kv_layout* layout, int64_t total_tokens,
                                        const gqla_hw* hw, gqla_path_estimate* est) {
  if (!est) return GQLA_ERR_INVALID_ARG;
  Problem pa, pg;
  gqla_status s = make_problem(dims, layout, 0, GQLA_PATH_ABSORB, &pa);
  if (s != GQLA_OK) return s;
  s = make_problem(dims, layout, 0, GQLA_PATH_GQA, &pg);
  if (s != GQLA_OK) return s;
  if (total_tokens < (int64_t)layout->batch * dims->s_q ||
      total_tokens > (int64_t)layout->batch * layout->max_seq_len)
    return GQLA_ERR_INVALID_ARG;
  Rates r;
  r.sms = hw ? hw->sms : num_sms();
  const double hbm = hw ? hw->hbm_gbs : kDefaultHbmGbs;
  const double tc = hw ? hw->tc_tflops : kDefaultTcTflops;
  if (r.sms < 1 || !(hbm > 0.0) || !(tc > 0.0)) return GQLA_ERR_INVALID_ARG;
  r.bw = hbm * 1e3;              // GB/s -> bytes/us
  r.bw_sm = r.bw / r.sms;
  r.tc_sm = tc * 1e6 / r.sms;    // TFLOP/s -> flop/us
  est->absorb_us = absorb_us(pa, total_tokens, r);
  est->gqa_us = gqa_us(pg, total_tokens, r);
  est->path = est->gqa_us < est->absorb_us ? GQLA_PATH_GQA : GQLA_PATH_ABSORB;
  return GQLA_OK;
}
