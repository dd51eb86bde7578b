// psi_fast.cu - streaming pipeline of the sampled linear verify (T > 0) for
// 16-byte aligned rows.
//
// Sources (page title, section): "Uno Psi-Spec 是什麼？Diffusion-Augmented LLM
// 如何保留 AR 分布、一次驗證多個 Token" (alphalab.site), "Uno Psi-Spec 怎麼運作？
// 完整走一次四個 Token", steps 3-4 and the bonus paragraph (accept while
// u < p/q, longest accepted prefix, residual correction, bonus token);
// "想跑 Uno：先確認官方程式需要的環境" (temperature, top-p).
//
// Kernels, in launch order:
//   round_advance  (early-exit rounds only) One thread per sequence: lists
//              the rows and units of the next round of positions for the
//              sequences whose drafts were all accepted so far.
//   row_scan   (psi_scan.cu) Streams every listed logit row once from HBM:
//              per slice of a row, its maximum, its fp32 sum of
//              exponentials and its set-aside list (elements above the
//              running top-p threshold).
//   row_finish One CTA of four warps per listed row: row maximum, Z, the
//              top-p threshold and renormaliser from the slice records and
//              lists, exact
//              (double masses, 2^52 fixed-point sums); the row's candidates
//              compacted at the front of its list area.
//   unit       One thread per (sequence, position) unit: accepts or rejects
//              the drafted token from the two finished rows (p(x), q(x) in
//              double); a unit whose row failed is listed for the second pass.
//   row_scan / row_finish / unit, second pass   Rows whose window held less
//              than top_p of the mass (rescanned with a wider window) or
//              whose lists overflowed (rescanned with the exact maximum
//              known); once, after the last round.
//   (cluster kernel, list mode)  Units the second pass could not settle.
//   fast_emit  One warp per sequence: the first rejected position (a ballot
//              over the positions), the emitted tokens, and the position
//              whose token is still to be drawn, listed.
//   draw       One CTA per listed position: the correction (residual
//              max(0, p - q)) or bonus draw over p's nucleus, inverse CDF in
//              vocabulary order on exact integer sums.  Only the emitted
//              position of each sequence is drawn.
//   whole_row_draw  Without top-p (and top-k) the draw spans the vocabulary:
//              for rows of up to kWrMaxVocab entries, one CTA per such
//              position, from the rows' finished maxima and normalisers;
//              longer rows go to the cluster kernel in sample mode.  A call
//              launches either the draw kernel (top-p or top-k on) or the
//              whole-row draw, never both.
#include <algorithm>

#include "psi_finish.cuh"

namespace psi {

namespace {

using namespace finish;

constexpr int kListClusters = 16;
constexpr int kCounters = 10;  // work-list counters (see FastArgs::counters)
// Candidate window, in log2 units below the row maximum.  The first pass uses
// a narrow window (13 units for top_p <= 0.95, wider as top_p approaches 1);
// the second pass the wide one.
constexpr float kWindowBaseLog2 = 13.f;
constexpr float kWindowWideLog2 = 20.f;

// ---------------------------------------------------------------------------
// row_finish: one CTA per listed row
// ---------------------------------------------------------------------------
template <typename Bits>
__global__ void __launch_bounds__(kFinThreads) row_finish_kernel(const __grid_constant__ FastArgs a) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  __shared__ FinShared fsh;
  const int64_t R = a.rlist ? (int64_t)*a.rcount : a.rows;
  for (int64_t item = blockIdx.x; item < R; item += gridDim.x) {
    const int64_t r = a.rlist ? (int64_t)(a.rlist[item] & ~kWideBit) : item;
    const RowFin f = finish_row_cta<Bits>(a, r, fsh);
    if (threadIdx.x == 0) a.rfin[r] = f;
    __syncthreads();  // the shared lists are rewritten for the next row
  }
}

// ---------------------------------------------------------------------------
// unit: one thread per (sequence, position) unit: accept or reject
// ---------------------------------------------------------------------------
constexpr int kUnitThreads = 128;
constexpr int32_t kTokenDraw = -3;        // rec.token: the nucleus draw kernel decides it
constexpr int32_t kTokenWholeRow = -2;    // rec.token: a whole-row draw (no top-p)

__device__ __forceinline__ RowFin empty_fin() {
  RowFin f;
  f.m = -INFINITY;
  f.zp = 0.0;
  f.tau_bits = 0u;
  f.tau_key = 0u;
  f.n = 0;
  f.status = 0;
  f.pad = 0;
  return f;
}

template <typename Bits>
__global__ void __launch_bounds__(kUnitThreads) unit_kernel(const __grid_constant__ FastArgs a) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  const SampledArgs &s = a.s;
  const int32_t B = s.B, N = s.N, V = s.V;
  const int64_t n_items = a.ulist ? (int64_t)*a.ucount : (int64_t)N * (B + 1);
  for (int64_t item = (int64_t)blockIdx.x * kUnitThreads + threadIdx.x; item < n_items;
       item += (int64_t)gridDim.x * kUnitThreads) {
    const int64_t unit = a.ulist ? (int64_t)a.ulist[item] : item;
    const int32_t n = (int32_t)(unit / (B + 1)), i = (int32_t)(unit % (B + 1));
    const bool has_q = i < B;
    const int64_t rp_idx = unit;
    const int64_t rq_idx = (int64_t)N * (B + 1) + (int64_t)n * B + i;
    const RowFin fp = a.rfin[rp_idx];
    const RowFin fq = has_q ? a.rfin[rq_idx] : empty_fin();
    const int fail_q = fq.status & (kFinOverflow | kFinCoverage | kFinTopK);
    const int fail_p = fp.status & (kFinOverflow | kFinCoverage | kFinTopK);
    if (a.top_k > 0 && (((fp.status | fq.status) & kFinTopK) || ((fail_q || fail_p) && a.pass == 2))) {
      // the candidates do not hold a top-k set (or a rescan did not settle
      // the unit): the whole-row top-k path decides it at the end
      a.list_k[atomicAdd(&a.counters[9], 1)] = (int32_t)unit;
      a.rec[unit].accept = -1;  // a later round treats it as accepted
      continue;
    }
    if (fail_q || fail_p) {
      if (a.pass == 1) {  // rescan the failed rows, then finish the unit again
        // the rescan starts from the row maximum found here, so its
        // threshold is final from the first stage
        if (fail_q) {
          a.known_max[rq_idx] = fq.m;
          a.wide_rows[atomicAdd(&a.counters[2], 1)] =
              (int32_t)rq_idx | ((fail_q & kFinCoverage) ? kWideBit : 0);
        }
        if (fail_p) {
          a.known_max[rp_idx] = fp.m;
          a.wide_rows[atomicAdd(&a.counters[2], 1)] =
              (int32_t)rp_idx | ((fail_p & kFinCoverage) ? kWideBit : 0);
        }
        a.wide_units[atomicAdd(&a.counters[3], 1)] = (int32_t)unit;
        a.rec[unit].accept = -1;  // settled by the rescan; a later round treats it as accepted
      } else {  // the general path verifies this unit (records included)
        a.list_a[atomicAdd(&a.counters[0], 1)] = (int32_t)unit;
        a.rec[unit].accept = -1;  // decided at the end; a later round treats it as accepted
      }
      continue;
    }
    // ---- accept / reject the drafted token (double precision)
    const uint64_t seq = s.seq_ids ? s.seq_ids[n] : (uint64_t)n;
    int need = 1;
    if (has_q) {
      const Bits *row_p = static_cast<const Bits *>(s.ar) + unit * s.ar_stride;
      const Bits *row_q = static_cast<const Bits *>(s.draft) + ((int64_t)n * B + i) * s.draft_stride;
      const int32_t x = s.ids[(int64_t)n * B + i];
      double p = 0.0, q = 0.0;
      const bool valid = x >= 0 && x < V;
      if (valid) {
        const float xp = Elem<Bits>::to_float(row_p[x]);
        const float xq = Elem<Bits>::to_float(row_q[x]);
        if (xp >= Elem<Bits>::to_float(fp.tau_bits) && fp.zp > 0.0)
          p = exact_exp2d(xp, fp.m, a.coef64) / fp.zp;
        if (xq >= Elem<Bits>::to_float(fq.tau_bits) && fq.zp > 0.0)
          q = exact_exp2d(xq, fq.m, a.coef64) / fq.zp;
      }
      const double u = (double)uniform24(s.seed, seq, s.step, (uint64_t)i, PSI_PURPOSE_ACCEPT);
      const int accept = (u * q < p) ? 1 : 0;
      need = !accept;
      if (s.out_p) s.out_p[(int64_t)n * B + i] = (float)p;
      if (s.out_q) s.out_q[(int64_t)n * B + i] = (float)q;
      a.rec[unit].accept = accept;
      if (accept) a.rec[unit].token = -1;
      if (!valid && s.dev_status) atomicOr(s.dev_status, PSI_DEV_BAD_TOKEN_ID);
    } else {
      a.rec[unit].accept = 1;
    }
    if (((fp.status | fq.status) & kFinNonfinite) && s.dev_status)
      atomicOr(s.dev_status, PSI_DEV_NONFINITE);
    // the correction / bonus token: drawn after the emit step, and only for
    // the position each sequence emits
    if (need) a.rec[unit].token = a.use_window ? kTokenDraw : kTokenWholeRow;
  }
}

// ---------------------------------------------------------------------------
// draw: one CTA of kDrawWarps warps per listed unit (each sequence's emitted
// position)
// ---------------------------------------------------------------------------
constexpr int kDrawWarps = 4;
constexpr int kDrawThreads = kDrawWarps * 32;
constexpr int kDrawReg = kFinishCap / kDrawThreads;  // nucleus entries a thread searches
static_assert(kFinishCap % kDrawThreads == 0, "the nucleus fits the threads' registers");

struct DrawScratch {  // the CTA's shared memory: p's nucleus and its draw weights
  uint32_t idx[kFinishCap];
  unsigned long long w[kFinishCap];
  unsigned long long part[2][kDrawWarps];  // per-warp partial sums (two buffers)
};

// Sum over the CTA; every thread gets the total.  `buf` alternates between
// calls so that one barrier suffices.
__device__ __forceinline__ unsigned long long draw_block_sum(unsigned long long v,
                                                             DrawScratch *ds, int buf) {
  v = warp_sum_any(v);
  if ((threadIdx.x & 31) == 0) ds->part[buf][threadIdx.x >> 5] = v;
  __syncthreads();
  unsigned long long t = 0ull;
#pragma unroll
  for (int w = 0; w < kDrawWarps; ++w) t += ds->part[buf][w];
  return t;
}

template <typename Bits>
__global__ void __launch_bounds__(kDrawThreads) draw_kernel(const __grid_constant__ FastArgs a) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  __shared__ DrawScratch dsm;
  __shared__ int wcnt[kDrawWarps];
  DrawScratch *ds = &dsm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const SampledArgs &s = a.s;
  const int32_t B = s.B, N = s.N, V = s.V;
  const int64_t n_items = (int64_t)a.counters[8];
  int buf = 0;  // the partial-sum buffer of the next block sum
  for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int64_t unit = (int64_t)a.list_d[item];
    const int32_t n = (int32_t)(unit / (B + 1)), i = (int32_t)(unit % (B + 1));
    const bool has_q = i < B;
    const int64_t rp_idx = unit;
    const int64_t rq_idx = (int64_t)N * (B + 1) + (int64_t)n * B + i;
    const RowFin fp = a.rfin[rp_idx];
    const RowFin fq = has_q ? a.rfin[rq_idx] : empty_fin();
    const uint64_t seq = s.seq_ids ? s.seq_ids[n] : (uint64_t)n;
    const Bits *row_q =
        has_q ? static_cast<const Bits *>(s.draft) + ((int64_t)n * B + i) * s.draft_stride : nullptr;
    const float tau_q = Elem<Bits>::to_float(fq.tau_bits);
    // ---- correction / bonus draw over p's nucleus (its candidates with x >=
    // tau, compacted at the front of the p row's area), inverse CDF in
    // vocabulary order, exact integer sums
    const unsigned long long *pc =
        reinterpret_cast<const unsigned long long *>(a.cand + rp_idx * (int64_t)kCandCap);
    const int nc = (fp.status & kFinNonfinite) ? 0 : fp.n;
    const double inv_sp = 1.0 / (fp.zp * kFix52);  // p's nucleus mass in fixed-point units
    const double inv_zq = fq.zp > 0.0 ? 1.0 / fq.zp : 0.0;
    // p's nucleus with its masses (as weights) to the scratch, in any order
    // (the search below sums by vocabulary index)
    auto load_nucleus = [&]() -> int {
      int nn = 0;
      for (int base = 0; base < nc; base += kDrawThreads * kLoadChunk) {
        unsigned long long e[kLoadChunk];  // loads in flight together
#pragma unroll
        for (int h = 0; h < kLoadChunk; ++h) {
          const int j = base + kDrawThreads * h + tid;
          e[h] = j < nc ? __ldcg(pc + j) : 0ull;
        }
        uint32_t inm = 0u;  // bit h: entry h is in the nucleus
#pragma unroll
        for (int h = 0; h < kLoadChunk; ++h) {
          const int j = base + kDrawThreads * h + tid;
          const bool in = j < nc && Elem<Bits>::key((uint32_t)(e[h] >> 32)) >= fp.tau_key;
          inm |= (in ? 1u : 0u) << h;
        }
        const int cnt = __popc(inm);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += v;
        }
        if (lane == 31) wcnt[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kDrawWarps; ++w) {
          before += w < warp ? wcnt[w] : 0;
          total += wcnt[w];
        }
        int d = nn + before + incl - cnt;
        nn += total;
#pragma unroll
        for (int h = 0; h < kLoadChunk; ++h)
          if ((inm >> h) & 1u) {
            ds->idx[d] = (uint32_t)e[h];
            ds->w[d] = e[h] >> 32;  // the logit's bits until its mass replaces them
            ++d;
          }
        __syncthreads();  // wcnt is reused; the entries are complete
      }
#pragma unroll 4
      for (int j = tid; j < nn; j += kDrawThreads)
        ds->w[j] = fixed52(exact_exp2d(Elem<Bits>::to_float((uint32_t)ds->w[j]), fp.m, a.coef64));
      __syncthreads();
      return nn;
    };
    const int nn = load_nucleus();
    unsigned long long W = 0ull;
    if (has_q) {  // residual weights max(0, p - q), in double
      for (int base = 0; base < nn; base += kDrawThreads * kQChunk) {
        uint32_t xqb[kQChunk];  // q logits of the chunk, loads in flight together
#pragma unroll
        for (int c = 0; c < kQChunk; ++c) {
          const int j = base + kDrawThreads * c + tid;
          xqb[c] = j < nn ? (uint32_t)row_q[ds->idx[j]] : 0u;
        }
#pragma unroll
        for (int c = 0; c < kQChunk; ++c) {
          const int j = base + kDrawThreads * c + tid;
          if (j < nn) {
            const double pv = (double)ds->w[j] * inv_sp;
            const float xq = Elem<Bits>::to_float(xqb[c]);
            const double qv = xq >= tau_q ? exact_exp2d(xq, fq.m, a.coef64) * inv_zq : 0.0;
            const unsigned long long wj = pv > qv ? fixed52(fmin(pv - qv, 1.0)) : 0ull;
            ds->w[j] = wj;
            W += wj;
          }
        }
      }
      W = draw_block_sum(W, ds, buf);
      buf ^= 1;
      if (W == 0ull) load_nucleus();  // residual vanished: draw from p itself
    }
    if (W == 0ull) {
      for (int j = tid; j < nn; j += kDrawThreads) W += ds->w[j];
      W = draw_block_sum(W, ds, buf);
      buf ^= 1;
    }
    int32_t token = 0;
    if (W > 0ull) {
      // t = floor(u' * W) exactly (u' = k / 2^24); the token is the index
      // whose weight interval [C(x), C(x) + w_x) holds t, C(x) = weight of the
      // entries with index < x: the largest X with C(X) <= t, by bisection
      const float u2 = uniform24(s.seed, seq, s.step, (uint64_t)i, PSI_PURPOSE_RESID);
      const unsigned long long k = (unsigned long long)(u2 * 16777216.0f);
      const unsigned long long t = (__umul64hi(k, W) << 40) | ((k * W) >> 24);
      uint32_t ir[kDrawReg];
      unsigned long long wr[kDrawReg];
#pragma unroll
      for (int c = 0; c < kDrawReg; ++c) {
        const int j = tid + kDrawThreads * c;
        ir[c] = j < nn ? ds->idx[j] : 0xFFFFFFFFu;
        wr[c] = j < nn ? ds->w[j] : 0ull;
      }
      uint32_t lo = 0u, hi = (uint32_t)V;
      while (hi - lo > 1u) {
        const uint32_t mid = (lo + hi) >> 1;
        unsigned long long cm = 0ull;
#pragma unroll
        for (int c = 0; c < kDrawReg; ++c) cm += ir[c] < mid ? wr[c] : 0ull;
        cm = draw_block_sum(cm, ds, buf);
        buf ^= 1;
        if (cm > t) hi = mid;
        else lo = mid;
      }
      token = (int32_t)lo;
    }
    if (tid == 0) {
      a.rec[unit].token = token;
      s.out_tokens[unit] = token;
    }
    __syncthreads();  // the scratch is reused by the CTA's next unit
  }
}

// ---------------------------------------------------------------------------
// whole_row_draw: one CTA per listed position whose draw spans the whole
// vocabulary (no top-p and no top-k): the residual max(0, p - q) or p over
// every index, p and q from the rows' finished maxima and normalisers (the
// same ones the decision used), fp32 exponentials in 2^40 fixed point
// (order-free integer sums; the CDF is within ~1e-7 of the exact one),
// inverse CDF in vocabulary order.  Each warp sums a contiguous range of
// the vocabulary with coalesced loads; the range holding the draw's point
// is then split over every thread of the CTA (pieces of kWrPiece), a block
// scan finds the piece that holds it, and its thread walks the piece.
// ---------------------------------------------------------------------------
constexpr int kWrThreads = 512;
constexpr int kWrWarps = kWrThreads / 32;
constexpr int kWrPiece = 24;  // elements per thread in the final search
constexpr int32_t kWrMaxVocab = 16384;  // longest row drawn by one CTA
constexpr float kFix40f = 1099511627776.0f;  // 2^40

template <typename Bits>
__global__ void __launch_bounds__(kWrThreads) whole_row_draw_kernel(const __grid_constant__ FastArgs a) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  __shared__ unsigned long long wsum[kWrWarps];
  __shared__ int32_t token_sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const SampledArgs &s = a.s;
  const int32_t B = s.B, N = s.N, V = s.V;
  const int64_t n_items = (int64_t)a.counters[1];
  // warp w's range of the vocabulary: [w * span, (w + 1) * span)
  const int32_t span = (V + kWrWarps - 1) / kWrWarps;
  for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int64_t unit = (int64_t)a.list_b[item];
    const int32_t n = (int32_t)(unit / (B + 1)), i = (int32_t)(unit % (B + 1));
    const bool has_q = i < B;
    const RowFin fp = a.rfin[unit];
    const RowFin fq = has_q ? a.rfin[(int64_t)N * (B + 1) + (int64_t)n * B + i] : empty_fin();
    const uint64_t seq = s.seq_ids ? s.seq_ids[n] : (uint64_t)n;
    const Bits *row_p = static_cast<const Bits *>(s.ar) + unit * s.ar_stride;
    const Bits *row_q =
        has_q ? static_cast<const Bits *>(s.draft) + ((int64_t)n * B + i) * s.draft_stride : nullptr;
    const float shift_p = fp.m == -INFINITY ? -INFINITY : -fp.m * a.coef;
    const float shift_q = fq.m == -INFINITY ? -INFINITY : -fq.m * a.coef;
    const float inv_zp = fp.zp > 0.0 ? (float)(1.0 / fp.zp) : 0.f;
    const float inv_zq = fq.zp > 0.0 ? (float)(1.0 / fq.zp) : 0.f;
    int32_t token = 0;
    for (int pass = has_q ? 0 : 1; pass < 2; ++pass) {
      // explicit roundings: both searches below must see the same weights
      auto weight = [&](int32_t v) -> unsigned long long {
        float pv = __fmul_rn(fast_exp2(fmaf(Elem<Bits>::to_float((uint32_t)row_p[v]), a.coef, shift_p)), inv_zp);
        if (pass == 0)
          pv = __fmaf_rn(-fast_exp2(fmaf(Elem<Bits>::to_float((uint32_t)row_q[v]), a.coef, shift_q)), inv_zq, pv);
        return pv > 0.f ? __float2ull_rn(__fmul_rn(fminf(pv, 1.f), kFix40f)) : 0ull;
      };
      const int32_t w0 = warp * span, w1 = min(V, w0 + span);
      unsigned long long part = 0ull;
      for (int32_t v = w0 + lane; v < w1; v += 32) part += weight(v);
      part = warp_sum_any(part);
      if (lane == 0) wsum[warp] = part;
      __syncthreads();
      unsigned long long W = 0ull;
      for (int w = 0; w < kWrWarps; ++w) W += wsum[w];
      __syncthreads();
      if (W == 0ull) continue;  // no residual mass: draw from p
      const float u2 = uniform24(s.seed, seq, s.step, (uint64_t)i, PSI_PURPOSE_RESID);
      const unsigned long long k = (unsigned long long)(u2 * 16777216.0f);
      const unsigned long long t = (__umul64hi(k, W) << 40) | ((k * W) >> 24);
      // the warp whose range holds t, and the weight before that range
      int ws = 0;
      unsigned long long wb = 0ull;
      for (int w = 0; w < kWrWarps; ++w) {
        if (wb + wsum[w] > t) {
          ws = w;
          break;
        }
        wb += wsum[w];
      }
      if (tid == 0) token_sh = -1;
      __syncthreads();
      // that range split over every thread of the CTA, a chunk of
      // kWrThreads * kWrPiece elements at a time: contiguous pieces of
      // kWrPiece elements per thread, their loads in flight together
      const int32_t r1 = min(V, (ws + 1) * span);
      for (int32_t c0 = ws * span; c0 < r1; c0 += kWrThreads * kWrPiece) {
        const int32_t q0 = min(r1, c0 + tid * kWrPiece), q1 = min(r1, q0 + kWrPiece);
        unsigned long long wv[kWrPiece];
        unsigned long long ps = 0ull;
#pragma unroll
        for (int e = 0; e < kWrPiece; ++e) {
          wv[e] = q0 + e < q1 ? weight(q0 + e) : 0ull;
          ps += wv[e];
        }
        // exclusive scan of the pieces over the CTA
        unsigned long long incl = ps;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long x = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += x;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        unsigned long long lb = wb + incl - ps, chunk = 0ull;
        for (int w = 0; w < kWrWarps; ++w) {
          if (w < warp) lb += wsum[w];
          chunk += wsum[w];
        }
        if (lb <= t && t < lb + ps) {  // exactly one thread's piece holds t
          unsigned long long run = lb;
#pragma unroll
          for (int e = 0; e < kWrPiece; ++e) {
            run += wv[e];
            if (run > t) {
              token_sh = q0 + e;
              break;
            }
          }
        }
        wb += chunk;
        __syncthreads();
        if (token_sh >= 0) break;
      }
      token = token_sh >= 0 ? token_sh : r1 - 1;  // the sums are exact: always found
      __syncthreads();
      break;
    }
    if (tid == 0) {
      a.rec[unit].token = token;
      s.out_tokens[unit] = token;
    }
  }
}

// ---------------------------------------------------------------------------
// fast_emit: one thread per sequence.
// ---------------------------------------------------------------------------
static_assert(PSI_MAX_B <= 32, "fast_emit: one lane per drafted position");

__global__ void __launch_bounds__(128) fast_emit_kernel(const __grid_constant__ FastArgs a) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t n = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // one warp per sequence
  const SampledArgs &s = a.s;
  if (n >= s.N) return;
  const int32_t B = s.B;  // <= 32: lane i holds position i
  const UnitRecord *r = a.rec + n * (B + 1);
  // the first rejected position (positions past it may hold records of an
  // earlier call: only the lowest rejection counts, and every position
  // before it was decided in this call)
  const uint32_t rej = __ballot_sync(0xFFFFFFFFu, lane < B && !r[lane].accept);
  const int32_t L = rej ? __ffs(rej) - 1 : B;
  const int32_t t = r[L].token;
  int32_t *tok = s.out_tokens + n * (B + 1);
  for (int32_t i = lane; i <= B; i += 32) tok[i] = i < L ? s.ids[n * B + i] : (i == L ? t : -1);
  if (lane == 0) {
    s.out_n[n] = L + 1;
    if (t == kTokenWholeRow) a.list_b[atomicAdd(&a.counters[1], 1)] = (int32_t)(n * (B + 1) + L);
    else if (t == kTokenDraw) a.list_d[atomicAdd(&a.counters[8], 1)] = (int32_t)(n * (B + 1) + L);
  }
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// ---------------------------------------------------------------------------
// round_advance: one thread per sequence.  Early-exit rounds: round k covers
// positions [sampled_round_begin(k), sampled_round_begin(k + 1)) of B + 1.
// A sequence takes part in round k when every drafted token of the earlier
// rounds was accepted (a unit left to the second pass or the general path
// counts as accepted: its rows are then read although a rejection may make
// them unused).  The kernel lists the round's rows and units, and resets the
// lists that the next round fills.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) round_advance_kernel(const __grid_constant__ FastArgs a,
                                                            int k) {
  pdl_wait();  // the previous kernel's results are visible
  pdl_trigger();
  const int32_t n = blockIdx.x * blockDim.x + threadIdx.x;
  const SampledArgs &s = a.s;
  const int32_t B = s.B, N = s.N;
  if (n == 0) {
    a.counters[4 + 2 * ((k + 1) & 1)] = 0;  // the next round's lists
    a.counters[5 + 2 * ((k + 1) & 1)] = 0;
  }
  if (n >= N) return;
  const int32_t i0 = sampled_round_begin(k, B);
  const int32_t i1 = sampled_round_begin(k + 1, B);
  int act = 1;
  if (k > 0) {
    act = a.active[n];
    const UnitRecord *r = a.rec + (int64_t)n * (B + 1);
    for (int32_t i = sampled_round_begin(k - 1, B); act && i < i0; ++i)
      if (i < B && r[i].accept == 0) act = 0;
  }
  a.active[n] = act;
  if (!act || i0 >= i1) return;
  int32_t *rc = a.counters + 4 + 2 * (k & 1);
  const int32_t nu = i1 - i0;
  const int32_t nd = min(i1, B) - i0;  // draft rows (the bonus row has none)
  const int32_t su = atomicAdd(rc + 1, nu);
  const int32_t sr = atomicAdd(rc, nu + nd);
  for (int32_t i = i0; i < i1; ++i) {
    const int32_t unit = n * (B + 1) + i;
    a.round_units[su + (i - i0)] = unit;
    a.round_rows[sr + (i - i0)] = unit;  // the AR row has the unit's index
  }
  for (int32_t i = i0; i < i0 + nd; ++i)
    a.round_rows[sr + nu + (i - i0)] = N * (B + 1) + n * B + i;
}

template <typename Bits>
cudaError_t launch_fast_typed(const FastArgs &fa, const SampledPlan &plan, bool early_exit,
                              const KernelEvents &ev, cudaStream_t stream) {
  const int64_t units = (int64_t)fa.s.N * (fa.s.B + 1);
  const int64_t persistent = (int64_t)device_sm_count() * 8;
  const int64_t grid_unit = std::min<int64_t>((units + kUnitThreads - 1) / kUnitThreads, persistent);
  const int64_t grid_draw = std::min<int64_t>(fa.s.N, persistent);
  const int64_t grid_finish = std::min<int64_t>(fa.rows, (int64_t)device_sm_count() * 8);
  cudaError_t e;
  static DeviceOnce configure;  // carveouts, once per device
  e = configure([] {
    cudaError_t err = prefer_max_shared(draw_kernel<Bits>);
    if (err == cudaSuccess) err = prefer_max_shared(row_finish_kernel<Bits>);
    if (err == cudaSuccess) err = prefer_max_shared(round_advance_kernel);
    if (err == cudaSuccess) err = prefer_max_shared(fast_emit_kernel);
    return err;
  });
  if (e != cudaSuccess) return e;
  // the work-list counters of this call start at zero
  if ((e = cudaMemsetAsync(fa.counters, 0, kCounters * sizeof(int32_t), stream)) != cudaSuccess)
    return e;
  // rows / units of one pass (first scan or rescan), then finish them
  auto scan_and_finish = [&](const FastArgs &f, bool timed) -> cudaError_t {
    cudaError_t err;
    if (timed && ev.before && (err = cudaEventRecord(ev.before, stream)) != cudaSuccess) return err;
    if ((err = launch_row_scan(f, sizeof(Bits) == 2 ? PSI_DTYPE_BF16 : PSI_DTYPE_F32, stream)) !=
        cudaSuccess)
      return err;
    if (timed && ev.after && (err = cudaEventRecord(ev.after, stream)) != cudaSuccess) return err;
    if ((err = launch_pdl(row_finish_kernel<Bits>, dim3((unsigned)grid_finish), dim3(kFinThreads),
                          0, stream, f)) != cudaSuccess)
      return err;
    return launch_pdl(unit_kernel<Bits>, dim3((unsigned)grid_unit), dim3(kUnitThreads), 0, stream,
                      f);
  };
  // the second pass over the rows and units a first pass could not settle
  // (usually none: the CTAs find empty lists and exit).  With early-exit
  // rounds it runs once, after the last round: a unit left to it counts as
  // accepted when the next round's sequences are chosen.
  FastArgs f2 = fa;
  f2.pass = 2;
  f2.rlist = fa.wide_rows;
  f2.rcount = fa.counters + 2;
  f2.ulist = fa.wide_units;
  f2.ucount = fa.counters + 3;
  if (!early_exit) {
    if ((e = scan_and_finish(fa, true)) != cudaSuccess) return e;
    if ((e = scan_and_finish(f2, false)) != cudaSuccess) return e;
  } else {
    const int rounds = round_count(fa.s.B, PSI_SAMPLED_SHORT_ROUNDS,
                                   PSI_SAMPLED_ROUND_POSITIONS);
    for (int k = 0; k < rounds; ++k) {
      if ((e = launch_pdl(round_advance_kernel, dim3((fa.s.N + 127) / 128), dim3(128), 0, stream,
                          fa, k)) != cudaSuccess)
        return e;
      FastArgs f1 = fa;
      f1.rlist = fa.round_rows;
      f1.rcount = fa.counters + 4 + 2 * (k & 1);
      f1.ulist = fa.round_units;
      f1.ucount = fa.counters + 5 + 2 * (k & 1);
      if ((e = scan_and_finish(f1, k == 0)) != cudaSuccess) return e;
    }
    // one second pass after the last round, over every round's failures
    if ((e = scan_and_finish(f2, false)) != cudaSuccess) return e;
  }
  const psi_dtype dt = sizeof(Bits) == 2 ? PSI_DTYPE_BF16 : PSI_DTYPE_F32;
  SampledArgs sa = fa.s;
  sa.records = fa.rec;
  if (fa.top_k > 0) {
    e = launch_topk_units(sa, dt, fa.list_k, fa.counters + 9,
                          std::min<int64_t>(units, (int64_t)device_sm_count() * 4), stream);
    if (e != cudaSuccess) return e;
  }
  const int clusters_a = (int)std::min<int64_t>(units, kListClusters);
  e = launch_cluster_list(sa, dt, plan, kClusterModeList, fa.list_a, fa.counters + 0, clusters_a,
                          stream);
  if (e != cudaSuccess) return e;
  if ((e = launch_pdl(fast_emit_kernel, dim3((fa.s.N + 3) / 4), dim3(128), 0, stream, fa)) !=
      cudaSuccess)
    return e;
  // a call's draws are all of one kind: over the nucleus when the window is
  // in use (top-p or top-k), else over the whole row
  if (fa.use_window)
    return launch_pdl(draw_kernel<Bits>, dim3((unsigned)grid_draw), dim3(kDrawThreads), 0, stream,
                      fa);
  // the whole-row draws (no top-p, no top-k): one CTA per draw for short
  // rows, where a cluster's launch and synchronisation cost more than the
  // row; a cluster per draw for long ones, which one SM reads too slowly
  if (fa.s.V <= kWrMaxVocab) {
    const int32_t grid_wr = std::max<int32_t>(1, std::min<int32_t>(fa.s.N, device_sm_count()));
    return launch_pdl(whole_row_draw_kernel<Bits>, dim3((unsigned)grid_wr), dim3(kWrThreads), 0,
                      stream, fa);
  }
  const int clusters_b = std::min(fa.s.N, kListClusters);
  return launch_cluster_list(sa, dt, plan, kClusterModeSample, fa.list_b, fa.counters + 1,
                             clusters_b, stream);
}

}  // namespace

cudaError_t launch_row_finish(const FastArgs &fa, psi_dtype dtype, cudaStream_t stream) {
  const int64_t grid = std::min<int64_t>(fa.rows, (int64_t)device_sm_count() * 8);
  if (dtype == PSI_DTYPE_BF16) {
    static DeviceOnce configure;
    cudaError_t e = configure([] { return prefer_max_shared(row_finish_kernel<uint16_t>); });
    if (e != cudaSuccess) return e;
    return launch_pdl(row_finish_kernel<uint16_t>, dim3((unsigned)std::max<int64_t>(grid, 1)),
                      dim3(kFinThreads), 0, stream, fa);
  } else {
    static DeviceOnce configure;
    cudaError_t e = configure([] { return prefer_max_shared(row_finish_kernel<uint32_t>); });
    if (e != cudaSuccess) return e;
    return launch_pdl(row_finish_kernel<uint32_t>, dim3((unsigned)std::max<int64_t>(grid, 1)),
                      dim3(kFinThreads), 0, stream, fa);
  }
}

FastLayout fast_layout(int32_t N, int32_t B) {
  FastLayout L;
  const int64_t units = (int64_t)N * (B + 1);
  const int64_t rows = units + (int64_t)N * B;
  size_t off = 0;
  L.rec_off = off;
  off = align256(off + sizeof(UnitRecord) * (size_t)units);
  L.srec_off = off;
  off = align256(off + sizeof(SliceRecord) * (size_t)rows * kMaxSlices);
  L.cand_off = off;
  off = align256(off + sizeof(uint64_t) * (size_t)rows * kCandCap);
  L.known_off = off;
  off = align256(off + sizeof(float) * (size_t)rows);
  L.rfin_off = off;
  off = align256(off + sizeof(RowFin) * (size_t)rows);
  L.counters_off = off;
  off = align256(off + sizeof(int32_t) * kCounters);
  L.list_a_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)units);
  L.list_b_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)N);
  L.list_d_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)N);
  L.list_k_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)units);
  L.wide_rows_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)rows);
  L.wide_units_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)units);
  L.round_rows_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)rows);
  L.round_units_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)units);
  L.active_off = off;
  off = align256(off + sizeof(int32_t) * (size_t)N);
  L.total = off;
  return L;
}

bool fast_path_fits(int32_t N, int32_t B) {
  // row indices travel in 30 bits of a second-pass list entry
  return (int64_t)N * (2 * (int64_t)B + 1) < (int64_t(1) << 30);
}

cudaError_t launch_sampled_fast(const SampledArgs &a, psi_dtype dtype, const SampledPlan &plan,
                                void *workspace, const KernelEvents &ev, cudaStream_t stream) {
  const FastLayout L = fast_layout(a.N, a.B);
  char *ws = static_cast<char *>(workspace);
  FastArgs fa;
  fa.s = a;
  fa.g = plan_scan(a.V, dtype == PSI_DTYPE_BF16 ? 2 : 4);
  fa.rows = (int64_t)a.N * (a.B + 1) + (int64_t)a.N * a.B;
  fa.coef64 = 1.4426950408889634 / (double)a.temperature;
  fa.coef = (float)fa.coef64;
  // first-pass window: 13 log2 units for top_p <= 0.95, one more unit for
  // every halving of the allowed tail mass beyond 5%, at most the wide window
  double wlog2 = kWindowBaseLog2;
  if (a.top_p < 1.0f && a.top_p > 0.95f) wlog2 += log2(0.05 / (1.0 - (double)a.top_p));
  if (wlog2 > kWindowWideLog2) wlog2 = kWindowWideLog2;
  fa.win_narrow = (float)(wlog2 / fa.coef64);
  fa.win_wide = (float)(kWindowWideLog2 / fa.coef64);
  fa.use_top_p = a.top_p < 1.0f ? 1 : 0;
  fa.top_k = a.top_k;
  fa.use_window = (fa.use_top_p || fa.top_k > 0) ? 1 : 0;
  fa.pass = 1;
  fa.rec = reinterpret_cast<UnitRecord *>(ws + L.rec_off);
  fa.srec = reinterpret_cast<SliceRecord *>(ws + L.srec_off);
  fa.cand = reinterpret_cast<uint64_t *>(ws + L.cand_off);
  fa.known_max = reinterpret_cast<float *>(ws + L.known_off);
  fa.rfin = reinterpret_cast<RowFin *>(ws + L.rfin_off);
  fa.counters = reinterpret_cast<int32_t *>(ws + L.counters_off);
  fa.list_a = reinterpret_cast<int32_t *>(ws + L.list_a_off);
  fa.list_b = reinterpret_cast<int32_t *>(ws + L.list_b_off);
  fa.list_d = reinterpret_cast<int32_t *>(ws + L.list_d_off);
  fa.list_k = reinterpret_cast<int32_t *>(ws + L.list_k_off);
  fa.wide_rows = reinterpret_cast<int32_t *>(ws + L.wide_rows_off);
  fa.wide_units = reinterpret_cast<int32_t *>(ws + L.wide_units_off);
  fa.round_rows = reinterpret_cast<int32_t *>(ws + L.round_rows_off);
  fa.round_units = reinterpret_cast<int32_t *>(ws + L.round_units_off);
  fa.active = reinterpret_cast<int32_t *>(ws + L.active_off);
  fa.rlist = nullptr;
  fa.rcount = nullptr;
  fa.ulist = nullptr;
  fa.ucount = nullptr;
  fa.s.records = fa.rec;
  // without p / q outputs only the rows up to each sequence's first rejection
  // matter: verify in early-exit rounds
  const bool early_exit = a.out_p == nullptr && a.out_q == nullptr && a.N >= PSI_EARLY_EXIT_MIN_N;
  if (dtype == PSI_DTYPE_BF16) return launch_fast_typed<uint16_t>(fa, plan, early_exit, ev, stream);
  return launch_fast_typed<uint32_t>(fa, plan, early_exit, ev, stream);
}

}  // namespace psi
