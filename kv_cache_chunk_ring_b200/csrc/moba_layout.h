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

// Query intervals that may read the key at kpos (at most two): a key of C_j is
// read by C_i for i >= j and by N_i for i > j; a key of N_j by N_j; a key of B
// by B.  Returns the count; unused entries are empty ([0, 0)).
KVCR_HD int moba_col_intervals(const MobaLay& l, int kpos, int* lo, int* hi) {
  int kk, ki, ks, ke;
  const int nc = l.n * l.c;
  moba_block(l, kpos, kk, ki, ks, ke);
  lo[0] = hi[0] = lo[1] = hi[1] = 0;
  if (kk == kBlkC) {
    lo[0] = ki * l.c;
    hi[0] = nc;
    if (ki + 1 < l.n) {
      lo[1] = nc + (ki + 1) * l.c;
      hi[1] = 2 * nc;
      return 2;
    }
    return 1;
  }
  if (kk == kBlkN) {
    lo[0] = ks;
    hi[0] = ke;
    return 1;
  }
  lo[0] = 2 * nc;
  hi[0] = l.L;
  return 1;
}

// Smallest query range [lo, hi) holding every query that may read a key of
// [c0, c1).
KVCR_HD void moba_col_bounds(const MobaLay& l, int c0, int c1, int& lo, int& hi) {
  int kk, ki, ks, ke;
  lo = l.L;
  hi = 0;
  for (int cp = c0; cp < c1; cp = ke) {
    moba_block(l, cp, kk, ki, ks, ke);
    int a[2], b[2];
    const int n = moba_col_intervals(l, cp, a, b);
    for (int t = 0; t < n; ++t) {
      if (a[t] < lo) lo = a[t];
      if (b[t] > hi) hi = b[t];
    }
  }
}

}  // namespace kvcr
