// Split-S decode attention: a few query rows (L * Hq/Hkv <= 8, e.g. one new
// token of the 4 query heads that share a key/value head) against a long
// key/value cache.  The khchao.com NN-lab page ("Arithmetic Intensity of
// Autoregressive Decoding") notes that each new token must read the whole
// cache, so this path is bound by HBM bandwidth, not by arithmetic: it streams
// K and V once with coalesced 16-byte loads and uses no tensor cores.
//
// Work split: one CTA per (key chunk, key/value head, batch).  Inside a CTA
//   phase 1  each group of G = E/8 lanes takes one key at a time, dots its 8
//            features with every query row, and reduces the R partial dots
//            across the G lanes with a transposed butterfly (each exchange
//            halves the number of live values, so R rows cost log2(G) + R - 1
//            shuffles instead of R log2(G)); base-2 logits go to shared memory;
//   phase 2  one warp per row: row maximum, p = 2^(logit - max), row sum;
//   phase 3  each lane group streams V rows and accumulates p * v in fp32;
//            the groups' partial sums are added through shared memory.
// A chunk's result is (O_s normalised, lse_s in base 2).  With more than one
// chunk a second kernel merges them:  lse = log2 sum_s 2^lse_s  and
// O = sum_s 2^(lse_s - lse) O_s  (the logsumexp-merge identity: each chunk's
// softmax restricted to its keys, reweighted by its share of the total).
//
// Paged caches: the same kernels read a row's keys and values from pages of a
// shared pool through its block table (kPaged).  Row b's keys are the first
// seq_lens[b] tokens of pages block_table[b][0], block_table[b][1], ... in
// table order; the hourtab.com xFormers retainer post ("Related retainer
// posts") recalls engines reading pages past a sequence's allocation and
// returning garbage with no error, so here every table entry is checked
// against the pool before use: an entry outside it drops that page's tokens
// and records error 32 in the decode error word, a length outside
// [0, max_pages * page_size] is clamped and records error 31.  No address
// outside the pool is ever formed.
#include "common.cuh"

namespace sdpa15 {

// Error word of the decode kernels (0 = none), read and cleared by
// decode_take_error().
__device__ int g_decode_error = 0;

// Block table of a paged cache (all zero for a contiguous one).
struct PagedArgs {
  const int32_t* table;  // [B][max_pages] page indices into the pool
  const int32_t* lens;   // [B] tokens per row
  int max_pages;
  int num_pages;         // pages in the pool
  int shift;             // log2(page_size)
};

constexpr int kDecThreads = 256;
constexpr int kDecChunkMax = 1024;  // keys per CTA at most
constexpr int kDecUnroll = 8;       // keys in flight per lane group

// Number of key chunks for a decode problem (also sizes the workspace).
int decode_splits(int B, int Hkv, int S) {
  const int units = B * Hkv;
  int n = (S + kDecChunkMax - 1) / kDecChunkMax;
  const int want = (148 * 8 + units - 1) / units;  // enough CTAs to fill 148 SMs
  const int max_useful = (S + 127) / 128;          // keep chunks >= 128 keys
  n = max(n, min(want, max_useful));
  return max(1, min(n, 1024));
}

template <typename T>
struct Vec8;  // 8 elements as one 16-byte load
template <>
struct Vec8<__half> {
  __device__ static void load(const __half* ptr, float (&f)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(ptr));
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) { float2 x = __half22float2(h[t]); f[2 * t] = x.x; f[2 * t + 1] = x.y; }
  }
  __device__ static uint4 raw(const __half* ptr) { return __ldcs(reinterpret_cast<const uint4*>(ptr)); }
  __device__ static void cvt(const uint4& u, float (&f)[8]) {
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) { float2 x = __half22float2(h[t]); f[2 * t] = x.x; f[2 * t + 1] = x.y; }
  }
};
template <>
struct Vec8<__nv_bfloat16> {
  __device__ static void load(const __nv_bfloat16* ptr, float (&f)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(ptr));
    cvt(u, f);
  }
  __device__ static uint4 raw(const __nv_bfloat16* ptr) { return __ldcs(reinterpret_cast<const uint4*>(ptr)); }
  __device__ static void cvt(const uint4& u, float (&f)[8]) {
    // bf16 -> f32 is a 16-bit left shift of the bit pattern.
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      f[2 * t] = __uint_as_float(w[t] << 16);
      f[2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
    }
  }
};

// Transposed butterfly over the G lanes of a group: on entry each lane holds R
// partial sums; on exit it holds the full sum of row `row` (replicated on
// G/R lanes when R < G).
template <int R, int G>
__device__ __forceinline__ float group_reduce_rows(float (&v)[R], int lane, int& row) {
  int base = 0;
  int c = R;
#pragma unroll
  for (int off = G / 2; off >= 1; off >>= 1) {
    const bool hi = (lane & off) != 0;
    if (c > 1) {
      const int half = c / 2;
#pragma unroll
      for (int t = 0; t < R / 2; ++t) {
        if (t < half) {
          const float send = hi ? v[t] : v[t + half];
          const float keep = hi ? v[t + half] : v[t];
          v[t] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      if (hi) base += half;
      c = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
  row = base;
  return v[0];
}

// kPage: 0 a contiguous cache; 1 a paged one (pages of 1, 2 or 4 tokens);
// 2 a paged one with pages of 8 tokens or more.
template <typename T, int E, int R, int kPage>
__global__ void __launch_bounds__(kDecThreads, (R <= 4 ? 3 : 2))
decode_split_kernel(Params p, int nsplit, int chunk, PagedArgs pg) {
  constexpr bool kPaged = kPage != 0;
  constexpr int G = E / 8;              // lanes per key row (16-byte slices)
  constexpr int KPW = 32 / G;           // keys per warp step
  constexpr int NKG = kDecThreads / G;  // lane groups per CTA
  constexpr int NW = kDecThreads / 32;
  extern __shared__ float smem[];
  float* lg = smem;  // [chunk][R] base-2 logits, then weights; reused for the reduction
  __shared__ float s_max[R], s_sum[R];
  __shared__ int s_flag[R];  // 1: NaN logit, 2: +inf logit
  // Paged: the pool index of each page this chunk touches (-1: an entry
  // outside the pool).
  __shared__ int s_page[kPaged ? kDecChunkMax + 2 : 1];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int S_b = p.S;
  if constexpr (kPaged) {
    const int len = __ldg(pg.lens + b);
    S_b = min(max(len, 0), p.S);  // p.S = max_pages * page_size
    if (S_b != len && tid == 0 && split == 0 && kvh == 0) atomicCAS(&g_decode_error, 0, 31);
  }
  const int s0 = split * chunk;
  const int s1 = min(S_b, s0 + chunk);
  const int n = max(0, s1 - s0);
  const int first_page = kPaged ? (s0 >> pg.shift) : 0;
  if constexpr (kPaged) {
    // The host keeps rows within 2^20 tokens, so a chunk holds at most 1024
    // keys and touches at most kDecChunkMax + 2 pages.
    const int count = n > 0 ? min(((s0 + n - 1) >> pg.shift) - first_page + 1, kDecChunkMax + 2) : 0;
    for (int i = tid; i < count; i += kDecThreads) {
      const int e = __ldg(pg.table + (int64_t)b * pg.max_pages + first_page + i);
      const bool ok = e >= 0 && e < pg.num_pages;
      if (!ok) atomicCAS(&g_decode_error, 0, 32);
      s_page[i] = ok ? e : -1;
    }
    __syncthreads();
  }
  // Paged: element offset of key/value token j of this chunk in the pool
  // (without the head and feature terms), or -1 when its page is not in it.
  auto token_offset = [&](int j, const int64_t* st) -> int64_t {
    const int tok = s0 + j;
    const int page = s_page[(tok >> pg.shift) - first_page];
    if (page < 0) return -1;
    return (int64_t)page * st[0] + (int64_t)(tok & ((1 << pg.shift) - 1)) * st[2];
  };
  const int gl = lane % G;                 // lane within its group
  const int kg = warp * KPW + lane / G;    // group index
  const int rows = p.group * p.L;          // live rows (<= R)
  // Contiguous cache: this batch row's keys; paged: the pool.
  auto chunk_base = [&](const void* base, const int64_t* st) -> const T* {
    const T* b0 = static_cast<const T*>(base) + kvh * st[1] + gl * 8;
    if constexpr (kPaged) return b0;
    else return b0 + b * st[0];
  };

  // Query rows: row r = (query head kvh*group + r / L, position r % L).
  float qf[R][8];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r < rows) {
      const int hq = kvh * p.group + r / p.L, l = r % p.L;
      const T* qp = static_cast<const T*>(p.q) + b * p.qs[0] + hq * p.qs[1] + (int64_t)l * p.qs[2] + gl * 8;
      Vec8<T>::load(qp, qf[r]);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[r][e] *= p.scale_log2;  // fold scale and log2(e)
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[r][e] = 0.f;
    }
  }

  // Phase 1: logits.
  const T* kbase = chunk_base(p.k, p.ks);
  // Dot products of a key with every query row, reduced over the key's lane
  // group; the lanes holding a row's sum write its base-2 logit.
  auto logit = [&](int j, const uint4& raw, bool dropped) {
    float kf[8];
    Vec8<T>::cvt(raw, kf);
    float d[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaf(qf[r][e], kf[e], a);
      d[r] = a;
    }
    int row;
    const float full = group_reduce_rows<R, G>(d, gl, row);
    // lanes holding a replica of the same row: the first one writes
    if (j < n && (gl % (G / R > 0 ? G / R : 1)) == 0) lg[j * R + row] = dropped ? -INFINITY : full;
  };
  if constexpr (kPaged) {
    // A lane group takes kDecUnroll consecutive keys: with pages of 8 or
    // more tokens (kPage 2; chunks start at multiples of 8) they share one
    // page, so the group looks its page up once.  The loop bound is
    // warp-uniform.
    for (int it0 = 0; it0 < n; it0 += NKG * kDecUnroll) {
      const int jg = it0 + kg * kDecUnroll;
      uint4 raw[kDecUnroll];
      const int64_t off0 = (kPage == 2 && jg < n) ? token_offset(jg, p.ks) : -1;
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) {
        const int j = jg + u;
        const int64_t off = kPage == 2 ? (off0 >= 0 ? off0 + (int64_t)u * p.ks[2] : -1)
                                       : (j < n ? token_offset(j, p.ks) : -1);
        if (j < n && off >= 0) raw[u] = Vec8<T>::raw(kbase + off);
        else raw[u] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) {
        const int j = jg + u;
        const bool dropped = kPage == 2 ? off0 < 0 : (j < n && s_page[((s0 + j) >> pg.shift) - first_page] < 0);
        logit(j, raw[u], dropped);
      }
    }
  } else {
    // The loop bound is warp-uniform (the shuffles below need every lane).
    for (int jb = warp * KPW; jb < n; jb += NKG * kDecUnroll) {
      const int j0 = jb + lane / G;
      uint4 raw[kDecUnroll];
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) {
        const int j = j0 + u * NKG;
        if (j < n) raw[u] = Vec8<T>::raw(kbase + (int64_t)(s0 + j) * p.ks[2]);
        else raw[u] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) logit(j0 + u * NKG, raw[u], false);
    }
  }
  __syncthreads();

  // Phase 2: per-row maximum, weights and sum (one warp per row).
  for (int r = warp; r < R; r += NW) {
    float mx = -INFINITY;
    int flag = 0;
    for (int j = lane; j < n; j += 32) {
      const float x = lg[j * R + r];
      if (isnan(x)) flag |= 1;
      else if (x == INFINITY) flag |= 2;
      mx = fmaxf(mx, x);
    }
    mx = warp_max(mx);
    flag = __reduce_or_sync(0xffffffffu, flag);
    float sum = 0.f;
    const bool finite_max = mx > -INFINITY && mx < INFINITY;
    for (int j = lane; j < n; j += 32) {
      const float w = finite_max ? exp2f(lg[j * R + r] - mx) : 0.f;
      lg[j * R + r] = w;
      sum += w;
    }
    sum = warp_sum(sum);
    if (lane == 0) { s_max[r] = mx; s_sum[r] = sum; s_flag[r] = flag; }
  }
  __syncthreads();

  // Phase 3: weighted sum of V rows.
  float acc[R][8];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
  const T* vbase = chunk_base(p.v, p.vs);
  auto accumulate = [&](int j, const uint4& raw) {
    if (j >= n) return;
    float vf[8];
    Vec8<T>::cvt(raw, vf);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float w = lg[j * R + r];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[r][e] = fmaf(w, vf[e], acc[r][e]);
    }
  };
  if constexpr (kPaged) {
    for (int it0 = 0; it0 < n; it0 += NKG * kDecUnroll) {
      const int jg = it0 + kg * kDecUnroll;
      uint4 raw[kDecUnroll];
      const int64_t off0 = (kPage == 2 && jg < n) ? token_offset(jg, p.vs) : -1;
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) {
        const int j = jg + u;
        const int64_t off = kPage == 2 ? (off0 >= 0 ? off0 + (int64_t)u * p.vs[2] : -1)
                                       : (j < n ? token_offset(j, p.vs) : -1);
        if (j < n && off >= 0) raw[u] = Vec8<T>::raw(vbase + off);
        else raw[u] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) accumulate(jg + u, raw[u]);
    }
  } else {
    for (int jb = warp * KPW; jb < n; jb += NKG * kDecUnroll) {
      const int j0 = jb + lane / G;
      uint4 raw[kDecUnroll];
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) {
        const int j = j0 + u * NKG;
        if (j < n) raw[u] = Vec8<T>::raw(vbase + (int64_t)(s0 + j) * p.vs[2]);
        else raw[u] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) accumulate(j0 + u * NKG, raw[u]);
    }
  }
  __syncthreads();  // weights no longer needed: reuse shared memory
  float* red = smem;  // [NKG][R][E]
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float4* dst = reinterpret_cast<float4*>(red + ((size_t)kg * R + r) * E + gl * 8);
    dst[0] = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    dst[1] = make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
  }
  __syncthreads();

  // Sum the groups and write this chunk's result.
  for (int idx = tid; idx < rows * E; idx += kDecThreads) {
    const int r = idx / E, c = idx - r * E;
    float s = 0.f;
#pragma unroll 4
    for (int g = 0; g < NKG; ++g) s += red[((size_t)g * R + r) * E + c];
    const int hq = kvh * p.group + r / p.L, l = r % p.L;
    const float mx = s_max[r], sum = s_sum[r];
    const int flag = s_flag[r];
    float o, lse2;
    if (flag) { o = NAN; lse2 = (flag & 1) ? NAN : INFINITY; }
    else if (!(mx > -INFINITY)) { o = 0.f; lse2 = -INFINITY; }
    else { o = s / sum; lse2 = mx + log2f(sum); }
    const int64_t row = ((int64_t)b * p.Hq + hq) * p.L + l;
    if (nsplit == 1) {
      T* op = static_cast<T*>(p.o) + b * p.os[0] + hq * p.os[1] + (int64_t)l * p.os[2];
      op[c] = from_f32<T>(o);
      if (c == 0) p.lse[row] = lse2 * kLn2;
    } else {
      const int64_t nrows = (int64_t)p.B * p.Hq * p.L;
      float* wo = static_cast<float*>(p.ws);
      float* wl = wo + (int64_t)nsplit * nrows * E;
      wo[((int64_t)split * nrows + row) * E + c] = o;
      if (c == 0) wl[(int64_t)split * nrows + row] = lse2;
    }
  }
}

// Merge the chunks of each row: one warp per row.
template <typename T, int E>
__global__ void __launch_bounds__(128)
decode_combine_kernel(Params p, int nsplit) {
  const int64_t nrows = (int64_t)p.B * p.Hq * p.L;
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= nrows) return;
  const float* wo = static_cast<const float*>(p.ws);
  const float* wl = wo + (int64_t)nsplit * nrows * E;
  float mx = -INFINITY;
  bool nan = false, pinf = false;
  for (int s = lane; s < nsplit; s += 32) {
    const float x = wl[(int64_t)s * nrows + row];
    if (isnan(x)) nan = true;
    else if (x == INFINITY) pinf = true;
    mx = fmaxf(mx, x);
  }
  mx = warp_max(mx);
  nan = __any_sync(0xffffffffu, nan);
  pinf = __any_sync(0xffffffffu, pinf);
  constexpr int PL = (E + 31) / 32;
  float acc[PL];
#pragma unroll
  for (int t = 0; t < PL; ++t) acc[t] = 0.f;
  float tot = 0.f;
  const bool ok = !nan && !pinf && mx > -INFINITY;
  if (ok) {
    for (int s = 0; s < nsplit; ++s) {
      const float w = exp2f(wl[(int64_t)s * nrows + row] - mx);
      tot += w;
      const float* src = wo + ((int64_t)s * nrows + row) * E;
#pragma unroll
      for (int t = 0; t < PL; ++t) {
        const int c = lane + 32 * t;
        if (c < E && w > 0.f) acc[t] = fmaf(w, src[c], acc[t]);
      }
    }
  }
  const int b = (int)(row / ((int64_t)p.Hq * p.L));
  const int rem = (int)(row - (int64_t)b * p.Hq * p.L);
  const int hq = rem / p.L, l = rem % p.L;
  T* op = static_cast<T*>(p.o) + b * p.os[0] + hq * p.os[1] + (int64_t)l * p.os[2];
  const float inv = ok ? 1.f / tot : 0.f;
#pragma unroll
  for (int t = 0; t < PL; ++t) {
    const int c = lane + 32 * t;
    if (c < E) op[c] = from_f32<T>((nan || pinf) ? NAN : acc[t] * inv);
  }
  if (lane == 0) {
    float lse;
    if (nan) lse = NAN;
    else if (pinf) lse = INFINITY;
    else if (!(mx > -INFINITY)) lse = -INFINITY;
    else lse = (mx + log2f(tot)) * kLn2;
    p.lse[row] = lse;
  }
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int L, int S, int Ev) {
  const int ns = decode_splits(B, Hkv, S);
  if (ns <= 1) return 0;
  const size_t nrows = (size_t)B * Hq * L;
  return (size_t)ns * nrows * ((size_t)Ev + 1) * sizeof(float);
}

template <typename T, int E, int R, int kPage>
static cudaError_t launch_decode_t(const Params& p, const PagedArgs& pg, cudaStream_t st, int* launches) {
  constexpr bool kPaged = kPage != 0;
  const int ns = decode_splits(p.B, p.Hkv, p.S);
  int chunk = (p.S + ns - 1) / ns;
  if (kPaged) chunk = (chunk + 7) & ~7;  // chunks start at multiples of 8 tokens (at most 1024 keys still)
  constexpr int G = E / 8;
  constexpr int NKG = kDecThreads / G;
  const size_t smem_lg = (size_t)chunk * R * sizeof(float);
  const size_t smem_red = (size_t)NKG * R * E * sizeof(float);
  const size_t smem = smem_lg > smem_red ? smem_lg : smem_red;
  auto kern = decode_split_kernel<T, E, R, kPage>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid(ns, p.Hkv, p.B);
  kern<<<grid, kDecThreads, smem, st>>>(p, ns, chunk, pg);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  *launches = 1;
  if (ns > 1) {
    const int64_t nrows = (int64_t)p.B * p.Hq * p.L;
    decode_combine_kernel<T, E><<<(unsigned)((nrows + 3) / 4), 128, 0, st>>>(p, ns);
    err = cudaGetLastError();
    *launches = 2;
  }
  return err;
}

template <typename T, int E, int kPage>
static cudaError_t launch_decode_e(const Params& p, const PagedArgs& pg, cudaStream_t st, int* launches) {
  const int rows = p.group * p.L;
  if (rows <= 1) return launch_decode_t<T, E, 1, kPage>(p, pg, st, launches);
  if (rows <= 2) return launch_decode_t<T, E, 2, kPage>(p, pg, st, launches);
  if (rows <= 4) return launch_decode_t<T, E, 4, kPage>(p, pg, st, launches);
  return launch_decode_t<T, E, 8, kPage>(p, pg, st, launches);
}

template <typename T, int kPage>
static cudaError_t launch_decode_d(const Params& p, const PagedArgs& pg, cudaStream_t st, int* launches) {
  switch (p.E) {
    case 64: return launch_decode_e<T, 64, kPage>(p, pg, st, launches);
    case 128: return launch_decode_e<T, 128, kPage>(p, pg, st, launches);
    default: return launch_decode_e<T, 256, kPage>(p, pg, st, launches);
  }
}

// Whether the decode kernel takes this problem (16-bit dtype, E = Ev in
// {64, 128, 256}, no mask, at most 8 rows per key/value head, 16-byte
// aligned rows).
bool decode_supported(const Params& p, int dtype) {
  if (dtype != SDPA_F16 && dtype != SDPA_BF16) return false;
  if (p.mask != SDPA_MASK_NONE) return false;
  if (p.E != p.Ev || (p.E != 64 && p.E != 128 && p.E != 256)) return false;
  if (p.group * p.L > 8 || p.S < 1) return false;
  const int64_t* strides[4] = {p.qs, p.ks, p.vs, p.os};
  for (int t = 0; t < 4; ++t)
    for (int d = 0; d < 3; ++d)
      if ((strides[t][d] * 2) % 16 != 0) return false;
  const void* ptrs[4] = {p.q, p.k, p.v, p.o};
  for (int t = 0; t < 4; ++t)
    if (reinterpret_cast<uintptr_t>(ptrs[t]) % 16 != 0) return false;
  return true;
}

cudaError_t launch_decode(const Params& p, int dtype, cudaStream_t st, int* launches) {
  const PagedArgs none = {nullptr, nullptr, 0, 0, 0};
  if (dtype == SDPA_F16) return launch_decode_d<__half, 0>(p, none, st, launches);
  return launch_decode_d<__nv_bfloat16, 0>(p, none, st, launches);
}

// Paged cache: p.k / p.v are the page pools with strides (page, head, token
// in page, feature), p.S = max_pages * page_size; decode_supported(p) holds.
cudaError_t launch_decode_paged(const Params& p, const int32_t* table, const int32_t* lens, int max_pages,
                                int num_pages, int page_shift, int dtype, cudaStream_t st, int* launches) {
  const PagedArgs pg = {table, lens, max_pages, num_pages, page_shift};
  if (page_shift >= 3) {
    if (dtype == SDPA_F16) return launch_decode_d<__half, 2>(p, pg, st, launches);
    return launch_decode_d<__nv_bfloat16, 2>(p, pg, st, launches);
  }
  if (dtype == SDPA_F16) return launch_decode_d<__half, 1>(p, pg, st, launches);
  return launch_decode_d<__nv_bfloat16, 1>(p, pg, st, launches);
}

// Reads and clears the decode kernels' error word.  Synchronous.
cudaError_t decode_take_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, g_decode_error, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(int));
}

}  // namespace sdpa15
