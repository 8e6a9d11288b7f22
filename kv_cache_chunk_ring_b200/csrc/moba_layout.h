// MoBA mask geometry, shared by the host library and the MoBA kernel.
//
// Sequence [C1..Cn | N1..Nn | B]: n clean chunks, n noisy chunks (chunk_tokens
// each) and one bidirectional block of n_bidir * chunk_tokens tokens.  Rule
// ("Infinite Worlds with Versatile Interactions", causal-pretraining
// paragraph: teacher-forcing mask with an appended fully bidirectional block;
// "Mix Forcing", "Mix the training modes"):
//   query in C_i reads C_j, j <= i;  query in N_i reads C_j, j < i, and N_i;
//   query in B reads all of B.
// The rule is constant on each (query block, key block) pair, so a tile's
// class follows from the blocks its rows and columns span.
#pragma once

#ifndef __CUDACC__
#define KVCR_HD inline
#else
#define KVCR_HD __host__ __device__ __forceinline__
#endif

namespace kvcr {

enum { kTileEmpty = 0, kTilePartial = 1, kTileFull = 2 };
enum { kBlkC = 0, kBlkN = 1, kBlkB = 2 };

struct MobaLay {
  int n;  // clean chunks = noisy chunks
  int c;  // tokens per chunk
  int m;  // chunks in the bidirectional block
  int L;  // (2n + m) * c
};

// Block of position pos: kind, index within the kind (B is one block), and its
// [start, end) token range.
KVCR_HD void moba_block(const MobaLay& l, int pos, int& kind, int& idx, int& start, int& end) {
  const int nc = l.n * l.c;
  if (pos < nc) {
    kind = kBlkC;
    idx = pos / l.c;
    start = idx * l.c;
    end = start + l.c;
  } else if (pos < 2 * nc) {
    kind = kBlkN;
    idx = (pos - nc) / l.c;
    start = nc + idx * l.c;
    end = start + l.c;
  } else {
    kind = kBlkB;
    idx = 0;
    start = 2 * nc;
    end = l.L;
  }
}

KVCR_HD bool moba_ok(int qk, int qi, int kk, int ki) {
  if (qk == kBlkC) return kk == kBlkC && ki <= qi;
  if (qk == kBlkN) return (kk == kBlkC && ki < qi) || (kk == kBlkN && ki == qi);
  return kk == kBlkB;
}

// Class of the tile x tile block (i, j); only in-range rows/columns count.
KVCR_HD int moba_classify(const MobaLay& l, int i, int j, int tile) {
  const int r0 = i * tile, c0 = j * tile;
  if (r0 >= l.L || c0 >= l.L) return kTileEmpty;
  const int r1 = r0 + tile < l.L ? r0 + tile : l.L;
  const int c1 = c0 + tile < l.L ? c0 + tile : l.L;
  bool any = false, all = true;
  int qk, qi, qs, qe, kk, ki, ks, ke;
  for (int rp = r0; rp < r1; rp = qe) {
    moba_block(l, rp, qk, qi, qs, qe);
    for (int cp = c0; cp < c1; cp = ke) {
      moba_block(l, cp, kk, ki, ks, ke);
      const bool ok = moba_ok(qk, qi, kk, ki);
      any = any || ok;
      all = all && ok;
    }
  }
  return all ? kTileFull : (any ? kTilePartial : kTileEmpty);
}

// Allowed key intervals of the queries in [r0, r1): appends up to 2 intervals
// per distinct query block to lo/hi (cap entries); returns the count.  Used
// for the bounding key range of a row tile and for its non-empty tile count.
KVCR_HD int moba_row_intervals(const MobaLay& l, int r0, int r1, int* lo, int* hi, int cap) {
  int n = 0;
  int qk, qi, qs, qe;
  const int nc = l.n * l.c;
  for (int rp = r0; rp < r1; rp = qe) {
    moba_block(l, rp, qk, qi, qs, qe);
    if (qk == kBlkC) {
      if (n < cap) { lo[n] = 0; hi[n] = (qi + 1) * l.c; ++n; }
    } else if (qk == kBlkN) {
      if (qi > 0 && n < cap) { lo[n] = 0; hi[n] = qi * l.c; ++n; }
      if (n < cap) { lo[n] = nc + qi * l.c; hi[n] = nc + (qi + 1) * l.c; ++n; }
    } else {
      if (n < cap) { lo[n] = 2 * nc; hi[n] = l.L; ++n; }
    }
  }
  return n;
}

// Smallest key range [lo, hi) holding every key a query of [r0, r1) may read.
KVCR_HD void moba_row_bounds(const MobaLay& l, int r0, int r1, int& lo, int& hi) {
  int qk, qi, qs, qe;
  const int nc = l.n * l.c;
  lo = l.L;
  hi = 0;
  for (int rp = r0; rp < r1; rp = qe) {
    moba_block(l, rp, qk, qi, qs, qe);
    int a, b;
    if (qk == kBlkC) { a = 0; b = (qi + 1) * l.c; }
    else if (qk == kBlkN) { a = qi > 0 ? 0 : nc; b = nc + (qi + 1) * l.c; }
    else { a = 2 * nc; b = l.L; }
    if (a < lo) lo = a;
    if (b > hi) hi = b;
  }
}

}  // namespace kvcr
