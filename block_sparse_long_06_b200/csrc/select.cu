// Block selection: sinks + local window + dynamic top-p over the residual
// candidates, capped at k_max, floored at k_min; ties to the lower block id.
// (SpotAttention, Methodology §3: reserved sink prefix and recency suffix,
//  nucleus selection on the residual distribution until the cumulative mass
//  reaches p, floor K_min; RTPurbo, Methodology §3 (dynamic top-p) and §5
//  (histogram thresholding instead of a sort); HGA, Central mechanism §2 for
//  the prefill diagonal block.)
//
// One CTA per row: decode row = (b, g); prefill row = (b, g, query block i). The
// row's p is that of its kv head when per-head values are given (RTPurbo,
// Methodology §1: local heads keep their reserved blocks only).
// The candidates form one contiguous id range [c0, c1) in both phases. Steps:
//  1. keys: 32-bit order keys (smaller key = higher score; -0 folded into +0,
//     NaN last) staged in shared memory; M = max score over the candidates;
//  2. radix select (4 passes x 8 bits, warp-aggregated shared-memory histograms,
//     integer counts only, so deterministic) of the key of the Kcap-th candidate,
//     Kcap = the largest dynamic count the caps allow; equal keys are taken in
//     ascending id order via a block-wide scan;
//  3. when 0 < p < 1: Z = sum of exp(S - M) over all candidates and W = the same
//     sum over the Kcap winners (fp64, fixed reduction trees). If W < p * Z no
//     prefix of the winners reaches p and all Kcap are kept (the common case when
//     K_max binds). Otherwise the winners are sorted by (key, id) with a bitonic
//     sort, their masses exp(S - M) are prefix-summed in fp64 along that order
//     (fixed order, deterministic) and the first prefix reaching p * Z is cut;
//  4. kept list = [0, c0) ++ ascending dynamic ids ++ [c1, end), -1 padded.
//
// Long decode rows (more than 2048 candidates: few rows, each long, as at 1M
// tokens) run on a cluster of up to 8 CTAs per row: each CTA holds a contiguous
// slice of the candidates, and the cluster combines its maxima, radix histograms,
// equal-key counts, masses and output offsets through distributed shared memory,
// always in rank order, so every CTA takes the same decisions. Each CTA pushes its
// values into every peer's shared memory before a cluster barrier (remote stores do
// not stall; remote loads would wait about a thousand cycles each), and the common
// path needs one barrier per radix pass plus three.
#include <cooperative_groups.h>

#include "bsa_common.cuh"
#include "bsa_internal.h"

namespace cg = cooperative_groups;

namespace bsa {
namespace {

constexpr int kHistCopies = 8;
constexpr int kMaxCluster = 8;    // CTAs per long decode row, at most

BSA_DEVFN uint32_t order_key(float s) {
  if (s != s) return 0xffffffffu;           // NaN: lowest priority
  s = s + 0.0f;                               // -0 -> +0
  uint32_t u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // ascending in s
  return ~u;                                  // ascending key = descending score
}
// The score of a key (exact; -0 comes back as +0 and NaN as a NaN), so the mass
// sums read the keys already in shared memory instead of the scores in global memory.
BSA_DEVFN float key_score(uint32_t key) {
  const uint32_t u = ~key;
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}


__host__ __device__ __forceinline__ int skew(int i) { return i + (i >> 5); }

// Keys of the scores S[0, n) into shared memory; returns this thread's max score. The
// loads of 8 rounds are issued before any is used (one dependent round trip to L2
// each would dominate the selection of a short row).
template <int NT>
BSA_DEVFN float load_keys(const float* S, int n, uint32_t* keys, int tid) {
  float lmax = -INFINITY;
  for (int t0 = 0; t0 < n; t0 += 8 * NT) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = t0 + u * NT + tid;
      v[u] = t < n ? S[t] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = t0 + u * NT + tid;
      if (t < n) {
        keys[skew(t)] = order_key(v[u]);
        if (v[u] == v[u]) lmax = fmaxf(lmax, v[u]);
      }
    }
  }
  return lmax;
}

// Adds the digit of one key to a shared-memory histogram. Pass 0 reads the top byte,
// which most keys share: equal digits of a warp are combined first (match.any). In
// later passes the digits are spread out and match.any would cost more than it
// saves (it was a third of a 128K row's selection), so each lane adds its own.
BSA_DEVFN void hist_add(uint32_t* h, uint32_t digit, int pass, int lane) {
  if (pass == 0) {
    const uint32_t peers = __match_any_sync(0xffffffffu, digit);
    if (digit < 256u && lane == __ffs(peers) - 1) atomicAdd(&h[digit], __popc(peers));
  } else if (digit < 256u) {
    atomicAdd(&h[digit], 1u);
  }
}

// Deterministic block reductions / scans (fixed tree for a fixed NT).
template <int NT, typename T, typename Op>
BSA_DEVFN T block_allreduce(T v, T* scratch, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  T r = scratch[0];
  for (int w = 1; w < NT / 32; ++w) r = op(r, scratch[w]);
  __syncthreads();
  return r;
}

// Exclusive scan of one value per thread in thread order; returns the prefix, sets total.
template <int NT, typename T>
BSA_DEVFN T block_exscan(T v, T* scratch, T& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  T base = T(0);
  for (int w = 0; w < warp; ++w) base += scratch[w];
  T tot = T(0);
  for (int w = 0; w < NT / 32; ++w) tot += scratch[w];
  total = tot;
  __syncthreads();
  return base + inc - v;
}

// Radix select over keys[skew(0 .. n)) (4 passes x 8 bits, warp-aggregated shared-memory
// histograms, integer counts only): returns the rem-th smallest key (1-based) and leaves
// in `rem` how many keys equal to it are among the rem smallest (every smaller key is).
template <int NT>
BSA_DEVFN uint32_t radix_kth(const uint32_t* keys, int n, int& rem, uint32_t* hist,
                             uint32_t* s_bucket_info) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0u, pmask = 0u;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int x = tid; x < kHistCopies * 256; x += NT) hist[x] = 0u;
    __syncthreads();
    uint32_t* h = hist + (warp % kHistCopies) * 256;
    for (int t0 = 0; t0 < n; t0 += NT) {
      const int t = t0 + tid;
      uint32_t digit = 256u;
      if (t < n) {
        const uint32_t k = keys[skew(t)];
        if ((k & pmask) == prefix) digit = (k >> shift) & 255u;
      }
      hist_add(h, digit, pass, lane);
    }
    __syncthreads();
    for (int x = tid; x < 256; x += NT) {
      uint32_t tot = 0;
      for (int c = 0; c < kHistCopies; ++c) tot += hist[c * 256 + x];
      hist[x] = tot;  // copy 0 now holds totals (other copies no longer needed)
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t part = 0;
      for (int q = 0; q < 8; ++q) part += hist[lane * 8 + q];
      uint32_t inc = part;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t nn = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += nn;
      }
      const uint32_t exc = inc - part;
      const bool here = (exc < static_cast<uint32_t>(rem)) && (inc >= static_cast<uint32_t>(rem));
      if (here) {
        uint32_t c = exc;
        int bsel = lane * 8;
        for (int q = 0; q < 8; ++q) {
          const uint32_t hq = hist[lane * 8 + q];
          if (c + hq >= static_cast<uint32_t>(rem)) {
            bsel = lane * 8 + q;
            break;
          }
          c += hq;
        }
        s_bucket_info[0] = static_cast<uint32_t>(bsel);
        s_bucket_info[1] = c;  // count strictly below the bucket
      }
    }
    __syncthreads();
    prefix |= s_bucket_info[0] << shift;
    pmask |= 255u << shift;
    rem -= static_cast<int>(s_bucket_info[1]);
    __syncthreads();
  }
  return prefix;
}

template <int NT>
__global__ void __launch_bounds__(NT) select_kernel(const SelectArgs a, int max_nc, int sort_n) {
  constexpr int NW = NT / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  // layout: [sort buffer: sort_n u64][keys: skew(max_nc) u32][hist: copies*256 u32]
  //         [flags: (max_nc+31)/32 u32][scratch]
  uint64_t* sbuf = reinterpret_cast<uint64_t*>(smem);
  uint32_t* keys = reinterpret_cast<uint32_t*>(sbuf + sort_n);
  uint32_t* hist = keys + skew(max_nc) + 1;
  uint32_t* flags = hist + kHistCopies * 256;
  const int nflag_words = (max_nc + 31) / 32;
  __shared__ double dscr[NW];
  __shared__ uint32_t s_bucket_info[2];
  __shared__ int s_hit;
  __shared__ float s_fscr[NW];
  __shared__ int s_iscr[NW];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  grid_dependency_wait();   // scores come from the scoring kernel

  // ---- row geometry -------------------------------------------------------
  int nbr, c0, c1;
  const float* S;
  int32_t* kept;
  int32_t* kcount;
  if (a.phase == BSA_PHASE_DECODE) {
    const int b = row / a.Hkv;
    int Tb = a.seq_lens ? a.seq_lens[b] : a.T;
    Tb = Tb < 0 ? 0 : (Tb > a.T ? a.T : Tb);
    nbr = (Tb + kBlock - 1) / kBlock;
    c0 = min(a.n_sink, nbr);
    c1 = max(c0, nbr - a.n_local);
    S = a.scores + static_cast<int64_t>(row) * a.nb_max;
  } else {
    // the query block's segment [b0, b1) (its diagonal block when seg_blocks = 1) is
    // kept; candidates are the earlier blocks outside the sinks and the n_local blocks
    // before the segment (PBS-Attn, Methodology §2 for permuted segments)
    const int i = row % a.nqb;
    const int b0 = (i / a.seg_blocks) * a.seg_blocks;
    nbr = min(b0 + a.seg_blocks, a.nqb);
    c0 = min(a.n_sink, b0);
    c1 = max(c0, b0 - a.n_local);
    S = a.scores + static_cast<int64_t>(row) * a.nqb;
  }
  kept = a.kept + static_cast<int64_t>(row) * a.max_kept;
  kcount = a.kept_count + row;
  const int nC = c1 - c0;

  // top-p of this row's kv head (local heads have p <= 0: reserved blocks only)
  const int g_row = a.phase == BSA_PHASE_DECODE ? row % a.Hkv : (row / a.nqb) % a.Hkv;
  const float ph = a.head_p ? a.head_p[g_row] : a.p;
  int kcap;  // largest number of dynamic blocks the caps allow
  const int kminC = min(a.k_min, nC);
  if (ph <= 0.f)
    kcap = kminC;
  else
    kcap = max(min(a.k_max, nC), kminC);
  const bool need_mass = (ph > 0.f) && (ph < 1.f) && kcap > 0;

  // ---- 1. keys and max ------------------------------------------------------
  const float lmax = load_keys<NT>(S + c0, nC, keys, tid);
  for (int w = tid; w < nflag_words; w += NT) flags[w] = 0u;
  const float M = block_allreduce<NT>(lmax, s_fscr, [](float x, float y) { return fmaxf(x, y); });

  // blocked ownership for the scans: thread t owns [t*E, min(nC, (t+1)*E))
  const int E = (nC + NT - 1) / NT;
  const int seg0 = min(nC, tid * E), seg1 = min(nC, seg0 + E);

  int kdyn = 0;
  if (kcap > 0 && kcap < nC) {
    // ---- 2. radix select of the kcap-th key ------------------------------------
    int rem = kcap;
    const uint32_t prefix = radix_kth<NT>(keys, nC, rem, hist, s_bucket_info);
    // keys < prefix are in; among keys == prefix take the `rem` lowest ids
    int neq = 0;
    for (int t = seg0; t < seg1; ++t) neq += (keys[skew(t)] == prefix);
    int tot_eq;
    int eq_base = block_exscan<NT>(neq, s_iscr, tot_eq);
    for (int t = seg0; t < seg1; ++t) {
      const uint32_t k = keys[skew(t)];
      bool in = k < prefix;
      if (k == prefix) in = (eq_base++ < rem);
      if (in) atomicOr(&flags[t >> 5], 1u << (t & 31));
    }
    kdyn = kcap;
  } else if (kcap > 0) {  // every candidate is within the caps
    for (int t = tid; t < nC; t += NT) atomicOr(&flags[t >> 5], 1u << (t & 31));
    kdyn = nC;
  }
  __syncthreads();

  // ---- 3. top-p cut inside the kcap winners ------------------------------------
  if (need_mass) {
    // total mass over the candidates (fp64, fixed order)
    double z = 0.0, wsum = 0.0;
    const double Md = static_cast<double>(M);
    const bool all_inf = !(M > -INFINITY);
    for (int t = seg0; t < seg1; ++t) {
      const float s = key_score(keys[skew(t)]);
      const double m = all_inf ? 1.0 : ((s == s) ? exp(static_cast<double>(s) - Md) : 0.0);
      z += m;
      if ((flags[t >> 5] >> (t & 31)) & 1u) wsum += m;
    }
    double Z = block_allreduce<NT>(z, dscr, [](double x, double y) { return x + y; });
    const double W = block_allreduce<NT>(wsum, dscr, [](double x, double y) { return x + y; });
    // the winners' whole mass stays below p: every winner is kept, no order is needed
    if (W < static_cast<double>(ph) * Z) goto emit;
    // compact winners in id order, then sort by (key, id)
    int nsel = 0;
    for (int t = seg0; t < seg1; ++t) nsel += (flags[t >> 5] >> (t & 31)) & 1u;
    int tot;
    int pos = block_exscan<NT>(nsel, s_iscr, tot);
    for (int t = seg0; t < seg1; ++t)
      if ((flags[t >> 5] >> (t & 31)) & 1u)
        sbuf[pos++] = (static_cast<uint64_t>(keys[skew(t)]) << 32) | static_cast<uint32_t>(t);
    for (int x = kdyn + tid; x < sort_n; x += NT) sbuf[x] = ~0ull;
    __syncthreads();
    for (int kk = 2; kk <= sort_n; kk <<= 1) {
      for (int j = kk >> 1; j > 0; j >>= 1) {
        for (int x = tid; x < sort_n; x += NT) {
          const int y = x ^ j;
          if (y > x) {
            const uint64_t u = sbuf[x], v = sbuf[y];
            const bool asc = (x & kk) == 0;
            if ((u > v) == asc) {
              sbuf[x] = v;
              sbuf[y] = u;
            }
          }
        }
        __syncthreads();
      }
    }
    // inclusive fp64 prefix of masses along the sorted order
    const int E2 = (kdyn + NT - 1) / NT;
    const int q0 = min(kdyn, tid * E2), q1 = min(kdyn, q0 + E2);
    double loc = 0.0;
    for (int x = q0; x < q1; ++x) {
      const float s = S[c0 + static_cast<int>(sbuf[x] & 0xffffffffu)];
      loc += all_inf ? 1.0 : ((s == s) ? exp(static_cast<double>(s) - Md) : 0.0);
    }
    double dtot;
    double run = block_exscan<NT>(loc, dscr, dtot);
    if (tid == 0) s_hit = 0x7fffffff;
    __syncthreads();
    const double target = static_cast<double>(ph) * Z;
    for (int x = q0; x < q1; ++x) {
      const float s = S[c0 + static_cast<int>(sbuf[x] & 0xffffffffu)];
      run += all_inf ? 1.0 : ((s == s) ? exp(static_cast<double>(s) - Md) : 0.0);
      if (run >= target) {
        atomicMin(&s_hit, x);
        break;
      }
    }
    __syncthreads();
    const int capC = min(a.k_max, nC);
    const int k = (s_hit != 0x7fffffff) ? max(min(s_hit + 1, capC), kminC) : kdyn;
    // re-flag the first k of the order
    for (int w = tid; w < nflag_words; w += NT) flags[w] = 0u;
    __syncthreads();
    for (int x = tid; x < k; x += NT) {
      const int t = static_cast<int>(sbuf[x] & 0xffffffffu);
      atomicOr(&flags[t >> 5], 1u << (t & 31));
    }
    kdyn = k;
    __syncthreads();
  }

emit:
  // ---- 4. kept list ----------------------------------------------------------
  int nsel = 0;
  for (int t = seg0; t < seg1; ++t) nsel += (flags[t >> 5] >> (t & 31)) & 1u;
  int tot;
  int pos = block_exscan<NT>(nsel, s_iscr, tot);
  for (int t = seg0; t < seg1; ++t)
    if ((flags[t >> 5] >> (t & 31)) & 1u) kept[c0 + pos++] = c0 + t;
  for (int x = tid; x < c0; x += NT) kept[x] = x;
  const int nlocal = nbr - c1;
  for (int x = tid; x < nlocal; x += NT) kept[c0 + tot + x] = c1 + x;
  const int count = c0 + tot + nlocal;
  for (int x = count + tid; x < a.max_kept; x += NT) kept[x] = -1;
  if (tid == 0) *kcount = count;
}

// Level-2 routing of a decode row (HGA, Central mechanism §2): the groups of
// group_size tokens of the row's dynamically kept blocks are the candidates, in
// ascending group id (the kept list is ascending); the k_groups of highest group
// score are kept (ties to the lower group id: equal keys in enumeration order), by
// the same radix select as the blocks. Sink and local entries keep every group. Out:
// one bitmask per kept-list entry (bit k = group k of the block), 0 past the count.
template <int NT>
__global__ void __launch_bounds__(NT) select_groups_kernel(const GroupSelectArgs a) {
  constexpr int NW = NT / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  // layout: [block ids: max_kept i32][keys: skew(max_cand) u32][hist: copies*256 u32][flags]
  int32_t* ids = reinterpret_cast<int32_t*>(smem);
  uint32_t* keys = reinterpret_cast<uint32_t*>(ids + a.max_kept);
  uint32_t* hist = keys + skew(a.max_cand) + 1;
  uint32_t* flags = hist + kHistCopies * 256;
  __shared__ uint32_t s_bucket_info[2];
  __shared__ int s_iscr[NW];

  const int tid = threadIdx.x;
  const int row = blockIdx.x;
  grid_dependency_wait();   // the kept lists come from the block selection

  const int b = row / a.Hkv;
  int Tb = a.seq_lens ? a.seq_lens[b] : a.T;
  Tb = Tb < 0 ? 0 : (Tb > a.T ? a.T : Tb);
  const int nbr = (Tb + kBlock - 1) / kBlock;
  const int c0 = min(a.n_sink, nbr);
  const int c1 = max(c0, nbr - a.n_local);
  const int gpb = kBlock / a.group_size;
  const uint32_t all = gpb == 32 ? 0xffffffffu : (1u << gpb) - 1u;
  const int32_t* kept = a.kept + static_cast<int64_t>(row) * a.max_kept;
  int32_t* out = a.kept_groups + static_cast<int64_t>(row) * a.max_kept;
  const int count = max(0, min(a.kept_count[row], a.max_kept));
  // the dynamic entries sit between the sink prefix and the local suffix
  int kdyn = max(0, count - c0 - (nbr - c1));
  if (kdyn * gpb > a.max_cand) {   // more dynamic entries than k_max: not a kept list
    report(a.status, BSA_DEV_BAD_KEPT);
    kdyn = a.max_cand / gpb;
  }
  for (int e = tid; e < kdyn; e += NT) {
    const int j = kept[c0 + e];
    const bool ok = j >= c0 && j < c1;
    if (!ok) report(a.status, BSA_DEV_BAD_KEPT);
    ids[e] = ok ? j : -1;
  }
  __syncthreads();
  // groups of the last block that start past the sequence do not exist; only the
  // last dynamic entry can be that block
  int ncand = kdyn * gpb;
  if (kdyn > 0 && ids[kdyn - 1] == nbr - 1)
    ncand -= gpb - (Tb - (nbr - 1) * kBlock + a.group_size - 1) / a.group_size;
  const int64_t ngr = static_cast<int64_t>(a.nb_max) * gpb;
  const float* Sg = a.group_scores + static_cast<int64_t>(row) * ngr;
  for (int t = tid; t < ncand; t += NT) {
    const int j = ids[t / gpb];
    // a rejected entry takes part with the lowest priority and is dropped below
    keys[skew(t)] = j >= 0 ? order_key(Sg[static_cast<int64_t>(j) * gpb + t % gpb]) : 0xffffffffu;
  }
  const int nflag_words = (ncand + 31) / 32;
  for (int w = tid; w < nflag_words; w += NT) flags[w] = 0u;
  __syncthreads();

  const int kg = min(a.k_groups, ncand);
  if (kg == ncand) {
    for (int t = tid; t < ncand; t += NT) atomicOr(&flags[t >> 5], 1u << (t & 31));
  } else if (kg > 0) {
    int rem = kg;
    const uint32_t prefix = radix_kth<NT>(keys, ncand, rem, hist, s_bucket_info);
    const int E = (ncand + NT - 1) / NT;
    const int seg0 = min(ncand, tid * E), seg1 = min(ncand, seg0 + E);
    int neq = 0;
    for (int t = seg0; t < seg1; ++t) neq += (keys[skew(t)] == prefix);
    int tot_eq;
    int eq_base = block_exscan<NT>(neq, s_iscr, tot_eq);
    for (int t = seg0; t < seg1; ++t) {
      const uint32_t k = keys[skew(t)];
      bool in = k < prefix;
      if (k == prefix) in = (eq_base++ < rem);
      if (in) atomicOr(&flags[t >> 5], 1u << (t & 31));
    }
  }
  __syncthreads();
  for (int e = tid; e < a.max_kept; e += NT) {
    uint32_t m = 0u;
    if (e < c0 || (e >= c0 + kdyn && e < count)) {
      m = all;   // sink and local blocks stay whole
    } else if (e < c0 + kdyn && ids[e - c0] >= 0) {
      for (int k = 0; k < gpb; ++k) {
        const int t = (e - c0) * gpb + k;
        if (t < ncand && ((flags[t >> 5] >> (t & 31)) & 1u)) m |= 1u << k;
      }
    }
    out[e] = static_cast<int32_t>(m);
  }
}

// Writes `v` into slot `slot` of the array `box` of every CTA of the cluster. The
// exchanges push rather than pull: remote stores do not stall the writer, and after
// the next cluster barrier every CTA reads the values from its own shared memory
// (a remote read costs about a thousand cycles).
template <typename T>
BSA_DEVFN void push_ranks(cg::cluster_group& cluster, T* box, int slot, int CL, T v) {
  for (int r = 0; r < CL; ++r) *cluster.map_shared_rank(box + slot, r) = v;
}

template <int NT>
__global__ void __launch_bounds__(NT) select_cluster_kernel(const SelectArgs a, int per_cta,
                                                            int sort_n) {
  constexpr int NW = NT / 32;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  extern __shared__ __align__(16) unsigned char smem[];
  // layout: [sort buffer: sort_n u64][winners: sort_n u64][keys: skew(per_cta) u32]
  //         [hist: copies*256 u32][flags: per_cta/32 u32]
  uint64_t* sbuf = reinterpret_cast<uint64_t*>(smem);
  uint64_t* wbuf = sbuf + sort_n;
  uint32_t* keys = reinterpret_cast<uint32_t*>(wbuf + sort_n);
  uint32_t* hist = keys + skew(per_cta) + 1;
  uint32_t* flags = hist + kHistCopies * 256;
  const int nflag_words = (per_cta + 31) / 32;
  __shared__ double dscr[NW];
  __shared__ uint32_t s_bucket_info[2];
  __shared__ int s_hit;
  __shared__ float s_fscr[NW];
  __shared__ int s_iscr[NW];
  // values each CTA publishes to the cluster
  // values the CTAs push to one another, slot = the writer's rank
  __shared__ float rx_max[kMaxCluster];
  __shared__ uint32_t rx_hist[2][kMaxCluster * 256];
  __shared__ int rx_eq[kMaxCluster], rx_sel[kMaxCluster];
  __shared__ double rx_z[kMaxCluster], rx_w[kMaxCluster];
  // values read by pull (rare path)
  __shared__ int pub_cnt, pub_k;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x / CL;
  // every CTA of the cluster must be running before another writes into its shared
  // memory: arrive now, wait just before the first push (the key loads run between)
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  grid_dependency_wait();   // scores come from the scoring kernel

  // ---- row geometry (decode rows) --------------------------------------------
  const int b = row / a.Hkv;
  int Tb = a.seq_lens ? a.seq_lens[b] : a.T;
  Tb = Tb < 0 ? 0 : (Tb > a.T ? a.T : Tb);
  const int nbr = (Tb + kBlock - 1) / kBlock;
  const int c0 = min(a.n_sink, nbr);
  const int c1 = max(c0, nbr - a.n_local);
  const float* S = a.scores + static_cast<int64_t>(row) * a.nb_max;
  int32_t* kept = a.kept + static_cast<int64_t>(row) * a.max_kept;
  const int nC = c1 - c0;
  const float ph = a.head_p ? a.head_p[row % a.Hkv] : a.p;
  const int kminC = min(a.k_min, nC);
  const int kcap = ph <= 0.f ? kminC : max(min(a.k_max, nC), kminC);
  const bool need_mass = (ph > 0.f) && (ph < 1.f) && kcap > 0;
  // this CTA's slice [lo, hi) of the candidates
  const int lo = min(nC, rank * per_cta), hi = min(nC, lo + per_cta), n = hi - lo;

  // ---- 1. keys and the local max (published with the first exchange) -----------
  float lmax = load_keys<NT>(S + c0 + lo, n, keys, tid);
  for (int w = tid; w < nflag_words; w += NT) flags[w] = 0u;
  lmax = block_allreduce<NT>(lmax, s_fscr, [](float x, float y) { return fmaxf(x, y); });
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (tid < CL) *cluster.map_shared_rank(&rx_max[rank], tid) = lmax;
  float M = -INFINITY;
  auto cluster_max = [&]() {
    for (int r = 0; r < CL; ++r) M = fmaxf(M, rx_max[r]);
  };

  const int E = (n + NT - 1) / NT;
  const int seg0 = min(n, tid * E), seg1 = min(n, seg0 + E);
  int kdyn = 0;
  if (kcap > 0 && kcap < nC) {
    // ---- 2. radix select of the kcap-th key over the cluster's histograms ------
    // One cluster barrier per pass: the published histograms alternate between two
    // buffers, so a pass never overwrites a copy that another CTA may still read.
    uint32_t prefix = 0u, pmask = 0u;
    int rem = kcap;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      uint32_t* rx = rx_hist[pass & 1];
      for (int x = tid; x < kHistCopies * 256; x += NT) hist[x] = 0u;
      __syncthreads();
      uint32_t* h = hist + (warp % kHistCopies) * 256;
      for (int t0 = 0; t0 < n; t0 += NT) {
        const int t = t0 + tid;
        uint32_t digit = 256u;
        if (t < n) {
          const uint32_t k = keys[skew(t)];
          if ((k & pmask) == prefix) digit = (k >> shift) & 255u;
        }
        hist_add(h, digit, pass, lane);
      }
      __syncthreads();
      for (int x = tid; x < 256; x += NT) {
        uint32_t tot = 0;
        for (int c = 0; c < kHistCopies; ++c) tot += hist[c * 256 + x];
        push_ranks(cluster, rx, rank * 256 + x, CL, tot);
      }
      cluster.sync();
      if (pass == 0) cluster_max();
      for (int x = tid; x < 256; x += NT) {
        uint32_t tot = 0;
        for (int r = 0; r < CL; ++r) tot += rx[r * 256 + x];
        hist[x] = tot;
      }
      __syncthreads();
      if (warp == 0) {
        uint32_t part = 0;
        for (int q = 0; q < 8; ++q) part += hist[lane * 8 + q];
        uint32_t inc = part;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t nn = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += nn;
        }
        const uint32_t exc = inc - part;
        const bool here = (exc < static_cast<uint32_t>(rem)) && (inc >= static_cast<uint32_t>(rem));
        if (here) {
          uint32_t c = exc;
          int bsel = lane * 8;
          for (int q = 0; q < 8; ++q) {
            const uint32_t hq = hist[lane * 8 + q];
            if (c + hq >= static_cast<uint32_t>(rem)) {
              bsel = lane * 8 + q;
              break;
            }
            c += hq;
          }
          s_bucket_info[0] = static_cast<uint32_t>(bsel);
          s_bucket_info[1] = c;
        }
      }
      __syncthreads();
      prefix |= s_bucket_info[0] << shift;
      pmask |= 255u << shift;
      rem -= static_cast<int>(s_bucket_info[1]);
    }
    // keys < prefix are in; among keys == prefix the `rem` lowest ids, counted
    // across the cluster in rank (= id) order
    int neq = 0;
    for (int t = seg0; t < seg1; ++t) neq += (keys[skew(t)] == prefix);
    int tot_eq;
    int eq_base = block_exscan<NT>(neq, s_iscr, tot_eq);
    if (tid < CL) *cluster.map_shared_rank(&rx_eq[rank], tid) = tot_eq;
    cluster.sync();
    for (int r = 0; r < rank; ++r) eq_base += rx_eq[r];
    for (int t = seg0; t < seg1; ++t) {
      const uint32_t k = keys[skew(t)];
      bool in = k < prefix;
      if (k == prefix) in = (eq_base++ < rem);
      if (in) atomicOr(&flags[t >> 5], 1u << (t & 31));
    }
    kdyn = kcap;
  } else {
    cluster.sync();   // the local maxima are visible
    cluster_max();
    if (kcap > 0) {
      for (int t = tid; t < n; t += NT) atomicOr(&flags[t >> 5], 1u << (t & 31));
      kdyn = nC;
    }
  }
  __syncthreads();

  // ---- 3. masses and winner counts, exchanged in one step ------------------------
  // Z = sum of exp(S - M) over the candidates and W = the same over the kcap winners
  // (fp64, fixed reduction trees, ranks added in order). If W < p * Z no prefix of
  // the winners reaches p and all of them are kept (the common case when K_max binds).
  const double Md = static_cast<double>(M);
  const bool all_inf = !(M > -INFINITY);
  double zl = 0.0, wl = 0.0;
  if (need_mass) {
    double z = 0.0, wsum = 0.0;
    for (int t = seg0; t < seg1; ++t) {
      const float s = key_score(keys[skew(t)]);
      const double m = all_inf ? 1.0 : ((s == s) ? exp(static_cast<double>(s) - Md) : 0.0);
      z += m;
      if ((flags[t >> 5] >> (t & 31)) & 1u) wsum += m;
    }
    zl = block_allreduce<NT>(z, dscr, [](double x, double y) { return x + y; });
    wl = block_allreduce<NT>(wsum, dscr, [](double x, double y) { return x + y; });
  }
  int nsel = 0;
  for (int t = seg0; t < seg1; ++t) nsel += (flags[t >> 5] >> (t & 31)) & 1u;
  int tot;
  int pos = block_exscan<NT>(nsel, s_iscr, tot);
  if (tid < CL) {
    *cluster.map_shared_rank(&rx_z[rank], tid) = zl;
    *cluster.map_shared_rank(&rx_w[rank], tid) = wl;
    *cluster.map_shared_rank(&rx_sel[rank], tid) = tot;
  }
  cluster.sync();
  double Z = 0.0, W = 0.0;
  int below = 0, all = 0;
  for (int r = 0; r < CL; ++r) {   // rank order: a fixed summation order
    Z += rx_z[r];
    W += rx_w[r];
    if (r < rank) below += rx_sel[r];
    all += rx_sel[r];
  }
  if (need_mass && !(W < static_cast<double>(ph) * Z)) {
    // the cut may fall inside the winners: rank 0 orders all of them
    int wpos = pos;
    for (int t = seg0; t < seg1; ++t)
      if ((flags[t >> 5] >> (t & 31)) & 1u)
        wbuf[wpos++] = (static_cast<uint64_t>(keys[skew(t)]) << 32) | static_cast<uint32_t>(lo + t);
    if (tid == 0) pub_cnt = tot;
    cluster.sync();
    if (rank == 0) {
      int off = 0;
      for (int r = 0; r < CL; ++r) {
        const int cr = *cluster.map_shared_rank(&pub_cnt, r);
        const uint64_t* src = cluster.map_shared_rank(wbuf, r);
        for (int x = tid; x < cr; x += NT) sbuf[off + x] = src[x];
        off += cr;
      }
      for (int x = off + tid; x < sort_n; x += NT) sbuf[x] = ~0ull;
      __syncthreads();
      for (int kk = 2; kk <= sort_n; kk <<= 1) {
        for (int j = kk >> 1; j > 0; j >>= 1) {
          for (int x = tid; x < sort_n; x += NT) {
            const int y = x ^ j;
            if (y > x) {
              const uint64_t u = sbuf[x], v = sbuf[y];
              const bool asc = (x & kk) == 0;
              if ((u > v) == asc) {
                sbuf[x] = v;
                sbuf[y] = u;
              }
            }
          }
          __syncthreads();
        }
      }
      const int E2 = (kdyn + NT - 1) / NT;
      const int q0 = min(kdyn, tid * E2), q1 = min(kdyn, q0 + E2);
      double loc = 0.0;
      for (int x = q0; x < q1; ++x) {
        const float s = S[c0 + static_cast<int>(sbuf[x] & 0xffffffffu)];
        loc += all_inf ? 1.0 : ((s == s) ? exp(static_cast<double>(s) - Md) : 0.0);
      }
      double dtot;
      double run = block_exscan<NT>(loc, dscr, dtot);
      if (tid == 0) s_hit = 0x7fffffff;
      __syncthreads();
      const double target = static_cast<double>(ph) * Z;
      for (int x = q0; x < q1; ++x) {
        const float s = S[c0 + static_cast<int>(sbuf[x] & 0xffffffffu)];
        run += all_inf ? 1.0 : ((s == s) ? exp(static_cast<double>(s) - Md) : 0.0);
        if (run >= target) {
          atomicMin(&s_hit, x);
          break;
        }
      }
      __syncthreads();
      const int capC = min(a.k_max, nC);
      if (tid == 0) pub_k = (s_hit != 0x7fffffff) ? max(min(s_hit + 1, capC), kminC) : kdyn;
    }
    cluster.sync();
    const int k = *cluster.map_shared_rank(&pub_k, 0);
    for (int w = tid; w < nflag_words; w += NT) flags[w] = 0u;
    __syncthreads();
    const uint64_t* order = cluster.map_shared_rank(sbuf, 0);
    for (int x = tid; x < k; x += NT) {
      const int id = static_cast<int>(order[x] & 0xffffffffu);
      if (id >= lo && id < hi) atomicOr(&flags[(id - lo) >> 5], 1u << ((id - lo) & 31));
    }
    kdyn = k;
    cluster.sync();   // every flag is set; rank 0's order is no longer read
    // counts of the new winners
    nsel = 0;
    for (int t = seg0; t < seg1; ++t) nsel += (flags[t >> 5] >> (t & 31)) & 1u;
    pos = block_exscan<NT>(nsel, s_iscr, tot);
    if (tid == 0) pub_cnt = tot;
    cluster.sync();
    below = 0;
    all = 0;
    for (int r = 0; r < CL; ++r) {
      const int v = *cluster.map_shared_rank(&pub_cnt, r);
      if (r < rank) below += v;
      all += v;
    }
  }

  // ---- 4. kept list: each CTA's ids after those of the lower ranks ----------------
  for (int t = seg0; t < seg1; ++t)
    if ((flags[t >> 5] >> (t & 31)) & 1u) kept[c0 + below + pos++] = c0 + lo + t;
  if (rank == 0) {
    for (int x = tid; x < c0; x += NT) kept[x] = x;
    const int nlocal = nbr - c1;
    for (int x = tid; x < nlocal; x += NT) kept[c0 + all + x] = c1 + x;
    const int count = c0 + all + nlocal;
    for (int x = count + tid; x < a.max_kept; x += NT) kept[x] = -1;
    if (tid == 0) a.kept_count[row] = count;
  }
  cluster.sync();   // no CTA leaves while another may still read its shared memory
}

int pow2_at_least(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

template <int NT>
cudaError_t launch_nt(const SelectArgs& a, int rows, int max_nc, cudaStream_t s) {
  const int kcap_max = max(min(a.k_max, max_nc), min(a.k_min, max_nc));
  const int sort_n = pow2_at_least(max(kcap_max, 2));
  const int nflag_words = (max_nc + 31) / 32;
  size_t smem = static_cast<size_t>(sort_n) * 8 + (static_cast<size_t>(skew(max_nc)) + 1) * 4 +
                kHistCopies * 256 * 4 + (nflag_words + 1) * 4;
  smem = (smem + 15) & ~static_cast<size_t>(15);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(select_kernel<NT>, dim3(rows), dim3(NT), smem, s, a, max_nc, sort_n);
}

// Long decode rows: a cluster of CL = 2..8 CTAs per row, each with <= 4096 candidates.
template <int NT>
cudaError_t launch_cluster(const SelectArgs& a, int rows, int max_nc, cudaStream_t s) {
  int cl = 2;
  while (cl < 8 && cl * 2048 < max_nc) cl *= 2;
  const int per_cta = ((max_nc + cl - 1) / cl + 31) & ~31;
  const int kcap_max = max(min(a.k_max, max_nc), min(a.k_min, max_nc));
  const int sort_n = pow2_at_least(max(kcap_max, 2));
  const int nflag_words = (per_cta + 31) / 32;
  size_t smem = static_cast<size_t>(sort_n) * 16 + (static_cast<size_t>(skew(per_cta)) + 1) * 4 +
                kHistCopies * 256 * 4 + (nflag_words + 1) * 4;
  smem = (smem + 15) & ~static_cast<size_t>(15);
  cudaError_t e = cudaFuncSetAttribute(select_cluster_kernel<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * cl);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, select_cluster_kernel<NT>, a, per_cta, sort_n);
}

}  // namespace

cudaError_t launch_select_groups(const GroupSelectArgs& a, cudaStream_t s) {
  const int rows = a.B * a.Hkv;
  if (rows <= 0) return cudaSuccess;
  const size_t nflag_words = (a.max_cand + 31) / 32;
  size_t smem = static_cast<size_t>(a.max_kept) * 4 + (static_cast<size_t>(skew(a.max_cand)) + 1) * 4 +
                kHistCopies * 256 * 4 + (nflag_words + 1) * 4;
  smem = (smem + 15) & ~static_cast<size_t>(15);
  cudaError_t e = cudaFuncSetAttribute(select_groups_kernel<256>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(select_groups_kernel<256>, dim3(rows), dim3(256), smem, s, a);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  int rows, max_nc;
  if (a.phase == BSA_PHASE_DECODE) {
    rows = a.B * a.Hkv;
    max_nc = a.nb_max;
  } else {
    rows = a.B * a.Hkv * a.nqb;
    max_nc = a.nqb;
  }
  if (rows <= 0) return cudaSuccess;
  max_nc = max(max_nc, 1);
  if (a.phase == BSA_PHASE_DECODE && max_nc > 2048) {
    // few long rows: one cluster of CTAs per row
    return launch_cluster<256>(a, rows, max_nc, s);
  }
  if (max_nc <= 2048) return launch_nt<256>(a, rows, max_nc, s);
  if (max_nc <= 8192) return launch_nt<512>(a, rows, max_nc, s);
  return launch_nt<1024>(a, rows, max_nc, s);
}

}  // namespace bsa
