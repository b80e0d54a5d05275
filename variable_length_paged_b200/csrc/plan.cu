// plan.cu -- on-device work planners, rebuilt every decode step from seq_lens.
//
// "Tencent HPC lands in SGLang, challenging default inference kernels",
// section "Why Tencent HPC matters for online model serving": the KV-cache
// work is cut into uniform tiles and handed to CTAs by the current workload,
// and the mapping is rebuilt as request lengths change; the comparator is a
// static split-k schedule that idles units or launches empty chunks.
//
// Both planners run as one 256-thread CTA and write the same work list:
// segments {request, cta, tile_begin, tile_end} in global tile order, the
// per-request and per-CTA segment ranges, and a header.  Everything is integer
// arithmetic, so the result is bit-exact and independent of thread timing.
#include <algorithm>
#include <climits>

#include "append_rows.cuh"
#include "da_internal.cuh"
#include "host_inputs.cuh"

namespace da {
namespace {

constexpr int kPlanThreads = 256;  // few warps: the plan is latency-bound, every barrier counts
constexpr int kPlanWarps = kPlanThreads / 32;

// Exclusive block-wide scan of one value per thread; also returns the total.
__device__ int block_exclusive_scan(int v, int* total, int* warp_buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_buf[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int i = 0; i < kPlanWarps; ++i) {
    const int t = warp_buf[i];
    before += i < warp ? t : 0;
    all += t;
  }
  *total = all;
  __syncthreads();  // warp_buf may be reused by the next call
  return before + x - v;
}

// Tile count of one request; an out-of-range length counts as 0 and is reported.
__device__ int request_tiles(const PlanParams& p, int b, int* s_bad) {
  const int L = p.seq_lens[b];
  if (L < 0 || (int64_t)L > p.capacity_tokens) {
    atomicMin(s_bad, b);
    return 0;
  }
  return (int)(((int64_t)L + p.tile_tokens - 1) / p.tile_tokens);
}

// Prefix arrays are kept in shared memory when the batch fits, else read back
// from global memory (written by this block and visible after __syncthreads).
constexpr int kSmemBatch = 4096;

// Phase shared by both planners: req_tile_prefix and U (and the largest n_b).  Each
// non-empty request counts start_units more units than its tiles (the dynamic plan's start
// cost; 0 for the static plan), so the prefix and U are in units.
__device__ void tile_prefix(const PlanParams& p, int32_t* rtp, int32_t* s_rtp, int* warp_buf, int* s_bad, int* U,
                            int* max_tiles, int start_units) {
  int carry = 0, mx = 0;
  for (int base = 0; base < p.batch; base += kPlanThreads) {
    const int b = base + threadIdx.x;
    const int tiles = b < p.batch ? request_tiles(p, b, s_bad) : 0;
    const int n = tiles > 0 ? tiles + start_units : 0;
    int total;
    const int excl = block_exclusive_scan(n, &total, warp_buf);
    if (b < p.batch) {
      rtp[b + 1] = carry + excl + n;
      if (s_rtp) s_rtp[b + 1] = carry + excl + n;
    }
    carry += total;
    mx = max(mx, n);
  }
  if (threadIdx.x == 0) {
    rtp[0] = 0;
    if (s_rtp) s_rtp[0] = 0;
  }
  if (max_tiles) {  // block max of n (static plan only)
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) warp_buf[threadIdx.x >> 5] = mx;
    __syncthreads();
    int all = 0;
#pragma unroll
    for (int i = 0; i < kPlanWarps; ++i) all = max(all, warp_buf[i]);
    *max_tiles = all;
  }
  *U = carry;
  __syncthreads();
}

// balance: 1 the plan used a balance table, 0 none was given, -1 one was given but refused.
__device__ void write_header(const PlanParams& p, int32_t* hdr, int U, int S, int kind, int splits, int bad,
                             int balance = 0) {
  hdr[kHdrUnits] = U;
  hdr[kHdrSegments] = S;
  hdr[kHdrCtas] = p.num_ctas;
  hdr[kHdrTile] = p.tile_tokens;
  hdr[kHdrStatus] = bad != INT_MAX ? DA_DEV_BAD_SEQLEN : balance < 0 ? DA_DEV_BAD_BALANCE : DA_DEV_OK;
  hdr[kHdrBadIndex] = bad == INT_MAX ? -1 : bad;
  hdr[kHdrKind] = kind;
  hdr[kHdrBatch] = p.batch;
  hdr[kHdrMaxSegments] = p.max_segments;
  hdr[kHdrSplits] = splits;
  hdr[kHdrBalance] = balance > 0 ? 1 : 0;
  for (int i = kHdrBalance + 1; i < kHdrWords; ++i) hdr[i] = 0;
}

// Largest i in [0, n] with a[i] <= x, for a non-decreasing a[0..n] with a[0] <= x.
__device__ __forceinline__ int last_not_above(const int32_t* a, int n, int64_t x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// CTA that owns global unit u, and the first unit of CTA c.  Even split: the unique c with
// floor(c*U/C) <= u < floor((c+1)*U/C); every product is below C*(U+1), and when that fits
// in 32 bits (the common case) the divisions are done in 32-bit integers.  Weighted (a
// balance table, U >= C): the ranges start at F[c], kept in shared memory.
struct Split {
  int64_t U, C;
  bool narrow;
  const int32_t* F;  // weighted range starts F[0..C], or null
  __device__ Split(int64_t u, int64_t c, const int32_t* f)
      : U(u), C(c), narrow(c * (u + 1) < (int64_t(1) << 31)), F(f) {}
  __device__ __forceinline__ int owner(int64_t u) const {
    if (F) return last_not_above(F, (int)C, u);
    if (narrow) return (int)(((uint32_t)(u + 1) * (uint32_t)C - 1u) / (uint32_t)U);
    return (int)(((u + 1) * C - 1) / U);
  }
  __device__ __forceinline__ int64_t first(int64_t c) const {
    if (F) return F[c];
    if (narrow) return (int64_t)(((uint32_t)c * (uint32_t)U) / (uint32_t)C);
    return c * U / C;
  }
};

// The balance table's weights, if the table fits this plan: each thread keeps the weights of
// CTAs t, t + kPlanThreads, ... (loaded before the lengths, so the two loads overlap).
constexpr int kBalancePerThread = (kBalanceMaxCtas + kPlanThreads - 1) / kPlanThreads;
struct BalanceWeights {
  int32_t w[kBalancePerThread];
  bool given;  // a table pointer was given
};

__device__ __forceinline__ BalanceWeights load_balance(const PlanParams& p) {
  BalanceWeights bw;
  bw.given = p.balance != nullptr;
#pragma unroll
  for (int k = 0; k < kBalancePerThread; ++k) {
    const int c = threadIdx.x + k * kPlanThreads;
    bw.w[k] = bw.given && p.num_ctas <= kBalanceMaxCtas && c < p.num_ctas ? p.balance[kBalanceHeader + c] : 1;
  }
  return bw;
}

// Checks the table against the plan (header, weight range) and, when it fits and U >= C,
// writes the weighted range starts F[c] = c + floor((U - C) * W_c / W) for c = 0..C.
// Returns 1 (table used), 0 (no table) or -1 (table refused).  Block-wide: every thread calls.
__device__ int weighted_starts(const PlanParams& p, const BalanceWeights& bw, int U, int32_t* F, int* warp_buf,
                               int* s_flag) {
  if (!bw.given) return 0;
  const int C = p.num_ctas;
  if (threadIdx.x == 0) {
    const bool hdr_ok = C <= kBalanceMaxCtas && p.balance[0] == kBalanceMagic && p.balance[1] == C &&
                        p.balance[2] == p.num_kv_heads;
    *s_flag = hdr_ok ? 1 : -1;
  }
  __syncthreads();
  int bad = 0;
#pragma unroll
  for (int k = 0; k < kBalancePerThread; ++k)
    if (threadIdx.x + k * kPlanThreads < C && (bw.w[k] < 1 || bw.w[k] > kBalanceMaxWeight)) bad = 1;
  if (__syncthreads_or(bad) && threadIdx.x == 0) *s_flag = -1;
  __syncthreads();
  const int flag = *s_flag;
  if (flag < 0 || U < C) return flag;
  // exclusive prefix of the weights (each sum below 2^28), then the range starts
  int carry = 0, total = 0;
#pragma unroll
  for (int k = 0; k < kBalancePerThread; ++k) {
    const int c = threadIdx.x + k * kPlanThreads;
    const int v = c < C ? bw.w[k] : 0;
    const int excl = block_exclusive_scan(v, &total, warp_buf);
    if (c < C) F[c] = carry + excl;
    carry += total;
    if (k * kPlanThreads + kPlanThreads >= C) break;  // uniform over the block
  }
  __syncthreads();
  const int64_t W = carry;
  for (int c = threadIdx.x; c <= C; c += kPlanThreads) {
    const int64_t Wc = c < C ? F[c] : W;
    F[c] = (int32_t)(c + (int64_t)(U - C) * Wc / W);
  }
  __syncthreads();
  return 1;
}

// The dynamic plan, computed by one block of kPlanThreads threads.
__device__ void plan_dynamic_body(const PlanParams& p) {
  __shared__ int warp_buf[32];
  __shared__ int s_bad, s_bal;
  __shared__ int32_t s_rtp[kSmemBatch + 1], s_rsb[kSmemBatch + 1];
  __shared__ int32_t s_first[kBalanceMaxCtas + 1];
  const BalanceWeights bw = load_balance(p);
  if (threadIdx.x == 0) s_bad = INT_MAX;
  __syncthreads();

  const WsLayout L = ws_layout(p.batch, p.num_ctas, p.max_segments, p.num_kv_heads);
  int32_t* done = p.ws + L.req_done;
  for (int64_t i = threadIdx.x; i < (int64_t)p.batch * p.num_kv_heads; i += kPlanThreads) done[i] = 0;
  int32_t* hdr = p.ws + L.hdr;
  int4* segs = reinterpret_cast<int4*>(p.ws + L.segs);
  int32_t* rtp = p.ws + L.req_tile_prefix;
  int32_t* rsb = p.ws + L.req_seg_begin;
  int32_t* csb = p.ws + L.cta_seg_begin;
  const bool small = p.batch <= kSmemBatch;
  const int32_t* rtp_r = small ? s_rtp : rtp;
  const int32_t* rsb_r = small ? s_rsb : rsb;
  const int64_t C = p.num_ctas;

  // Units: every non-empty request's start units (a fixed cost charged to the CTA that
  // starts it), then its tiles; U counts both.  Request b's tiles are units [first_tile(b),
  // rtp[b + 1]).
  const int sc = p.start_cost;
  int U;
  tile_prefix(p, rtp, small ? s_rtp : nullptr, warp_buf, &s_bad, &U, nullptr, sc);
  const int balance = weighted_starts(p, bw, U, s_first, warp_buf, &s_bal);
  const Split sp(U, C, balance > 0 && (int64_t)U >= C ? s_first : nullptr);
  auto first_tile = [&](int b) -> int { return rtp_r[b] + (rtp_r[b + 1] > rtp_r[b] ? sc : 0); };

  // Segments per request.  With U >= C every CTA owns at least one unit, so a
  // request whose tiles span CTAs [cf, cl] has cl - cf + 1 segments.  With U < C each
  // CTA owns at most one unit, so every tile is its own segment.
  const bool sparse = (int64_t)U < C;
  int carry = 0;
  for (int base = 0; base < p.batch; base += kPlanThreads) {
    const int b = base + threadIdx.x;
    int ns = 0;
    if (b < p.batch) {
      const int p0 = first_tile(b), n = rtp_r[b + 1] - p0;
      if (n > 0) ns = sparse ? n : sp.owner(p0 + n - 1) - sp.owner(p0) + 1;
    }
    int total;
    const int excl = block_exclusive_scan(ns, &total, warp_buf);
    if (b < p.batch) {
      rsb[b + 1] = carry + excl + ns;
      if (small) s_rsb[b + 1] = carry + excl + ns;
    }
    carry += total;
  }
  if (threadIdx.x == 0) {
    rsb[0] = 0;
    if (small) s_rsb[0] = 0;
  }
  const int S = carry;
  __syncthreads();

  // One thread per segment: find its request, then its CTA and tile range.
  for (int s = threadIdx.x; s < S; s += kPlanThreads) {
    const int b = last_not_above(rsb_r, p.batch, s);  // rsb[b] <= s < rsb[b+1]
    const int j = s - rsb_r[b];
    const int p0 = first_tile(b), n = rtp_r[b + 1] - p0;
    if (sparse) {
      segs[s] = make_int4(b, sp.owner((int64_t)p0 + j), j, j + 1);
    } else {
      const int c = sp.owner(p0) + j;
      const int64_t lo = max((int64_t)p0, sp.first(c));
      const int64_t hi = min((int64_t)p0 + n, sp.first(c + 1));
      segs[s] = make_int4(b, c, (int)(lo - p0), (int)(hi - p0));
    }
  }
  // One thread per CTA: its first segment.  Request r holds CTA c's first unit u0; the
  // segments before CTA c's are those of the requests before r and, of r's, those of the CTAs
  // before c (dense: one per CTA from the owner of r's first tile on; sparse: one per tile
  // before u0).  A CTA whose units are all start units gets an empty range.
  for (int c = threadIdx.x; c <= p.num_ctas; c += kPlanThreads) {
    int first;
    const int64_t u0 = c < p.num_ctas ? sp.first(c) : (int64_t)U;
    if (u0 >= U) {  // the end (also every CTA of an empty batch)
      first = S;
    } else {
      const int r = last_not_above(rtp_r, p.batch, u0);
      const int p0 = first_tile(r);
      first = rsb_r[r] + (sparse ? (int)max((int64_t)0, u0 - p0) : max(0, c - sp.owner(p0)));
    }
    csb[c] = first;
  }
  if (threadIdx.x == 0) write_header(p, hdr, U, S, DA_PLAN_DYNAMIC, 0, s_bad, balance);
}

__global__ void __launch_bounds__(kPlanThreads) plan_dynamic_kernel(const PlanParams p) {
  grid_dependency_wait();    // seq_lens may come from the previous kernel in the stream
  grid_dependents_launch();  // let the decode kernel start its prologue
  plan_dynamic_body(p);
}

// One launch for the step's bookkeeping: block 0 plans while the other blocks write
// every request's new K/V rows into their pages, so the appends add no time to the
// plan's critical path.  The decode kernel waits for the whole grid.
__global__ void __launch_bounds__(kPlanThreads) plan_append_kernel(const PlanParams p, const AppendParams a) {
  grid_dependency_wait();
  grid_dependents_launch();
  if (blockIdx.x == 0) {
    plan_dynamic_body(p);
  } else {
    for (int b = blockIdx.x - 1; b < a.batch; b += gridDim.x - 1) append_request_rows(a, b, threadIdx.x, blockDim.x);
  }
}

// The static split-k plan, computed by one block of kPlanThreads threads.
__device__ void plan_static_body(const PlanParams& p) {
  __shared__ int warp_buf[32];
  __shared__ int s_bad;
  __shared__ int32_t s_rtp[kSmemBatch + 1];
  if (threadIdx.x == 0) s_bad = INT_MAX;
  __syncthreads();

  const WsLayout L = ws_layout(p.batch, p.num_ctas, p.max_segments, p.num_kv_heads);
  int32_t* done = p.ws + L.req_done;
  for (int64_t i = threadIdx.x; i < (int64_t)p.batch * p.num_kv_heads; i += kPlanThreads) done[i] = 0;
  int32_t* hdr = p.ws + L.hdr;
  int4* segs = reinterpret_cast<int4*>(p.ws + L.segs);
  int32_t* rtp = p.ws + L.req_tile_prefix;
  int32_t* rsb = p.ws + L.req_seg_begin;
  int32_t* csb = p.ws + L.cta_seg_begin;
  const bool small = p.batch <= kSmemBatch;
  const int32_t* rtp_r = small ? s_rtp : rtp;
  const int S = p.width;

  int U, max_tiles;
  tile_prefix(p, rtp, small ? s_rtp : nullptr, warp_buf, &s_bad, &U, &max_tiles, 0);
  const int chunk = (max_tiles + S - 1) / S;
  const int total = p.batch * S;
  for (int i = threadIdx.x; i < total; i += kPlanThreads) {
    const int b = i / S, s = i - b * S;
    const int n = rtp_r[b + 1] - rtp_r[b];
    const int64_t lo = min((int64_t)s * chunk, (int64_t)n), hi = min((int64_t)(s + 1) * chunk, (int64_t)n);
    segs[i] = make_int4(b, i, (int)lo, (int)hi);
  }
  for (int b = threadIdx.x; b <= p.batch; b += kPlanThreads) rsb[b] = b * S;
  for (int c = threadIdx.x; c <= total; c += kPlanThreads) csb[c] = c;
  if (threadIdx.x == 0) write_header(p, hdr, U, total, DA_PLAN_STATIC, S, s_bad);
}

__global__ void __launch_bounds__(kPlanThreads) plan_static_kernel(const PlanParams p) {
  grid_dependency_wait();
  grid_dependents_launch();
  plan_static_body(p);
}

// Copy units [first, n) with stride `stride`, four loads in flight per thread (host
// memory is a bus round trip away).
template <typename T>
__device__ __forceinline__ void strided_copy(const T* src, T* dst, int64_t n, int64_t first, int64_t stride) {
  int64_t i = first;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const T a = src[i], b = src[i + stride], c = src[i + 2 * stride], d = src[i + 3 * stride];
    dst[i] = a;
    dst[i + stride] = b;
    dst[i + 2 * stride] = c;
    dst[i + 3 * stride] = d;
  }
  for (; i < n; i += stride) dst[i] = src[i];
}

// One launch brings the step's inputs in from mapped host memory and plans: block 0
// copies the lengths to the device (all its loads in flight at once) and plans from
// that copy; the other blocks copy the block table and q.  The decode kernel waits for
// the whole grid.
template <int kKind>
__global__ void __launch_bounds__(kPlanThreads) plan_host_kernel(const PlanParams p, const HostInputs h) {
  grid_dependency_wait();  // the previous step's kernels may still read the device copies
  grid_dependents_launch();
  if (blockIdx.x == 0) {
    strided_copy(h.seq_lens_host, h.seq_lens_dev, (int64_t)p.batch, (int64_t)threadIdx.x, (int64_t)kPlanThreads);
    __syncthreads();  // the block's own global writes are visible to it after the barrier
    PlanParams pd = p;
    pd.seq_lens = h.seq_lens_dev;
    if constexpr (kKind == DA_PLAN_DYNAMIC)
      plan_dynamic_body(pd);
    else
      plan_static_body(pd);
    return;
  }
  const int64_t first = (int64_t)(blockIdx.x - 1) * kPlanThreads + threadIdx.x;
  const int64_t stride = (int64_t)(gridDim.x - 1) * kPlanThreads;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    if (k >= h.num_copies) break;
    const HostCopy& c = h.copies[k];
    strided_copy(static_cast<const int4*>(c.src), static_cast<int4*>(c.dst), c.n16, first, stride);
    strided_copy(reinterpret_cast<const int32_t*>(static_cast<const int4*>(c.src) + c.n16),
                 reinterpret_cast<int32_t*>(static_cast<int4*>(c.dst) + c.n16), c.n4, first, stride);
  }
}

}  // namespace

namespace {
template <typename K>
cudaError_t launch_planner(K kernel, const PlanParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(kPlanThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}
}  // namespace

cudaError_t launch_plan_dynamic(const PlanParams& p, cudaStream_t stream) {
  return launch_planner(plan_dynamic_kernel, p, stream);
}

cudaError_t launch_plan_static(const PlanParams& p, cudaStream_t stream) {
  return launch_planner(plan_static_kernel, p, stream);
}

cudaError_t launch_plan_host(const PlanParams& p, int kind, const HostInputs& h, cudaStream_t stream) {
  int64_t units = 0;
  for (int k = 0; k < h.num_copies; ++k) units = max(units, h.copies[k].n16 + h.copies[k].n4);
  const int64_t per_pass = 4 * kPlanThreads;  // units one block moves with four loads in flight
  const int blocks = (int)std::min<int64_t>(147, (units + per_pass - 1) / per_pass);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1 + (unsigned)std::max(blocks, 1), 1, 1);
  cfg.blockDim = dim3(kPlanThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (kind == DA_PLAN_DYNAMIC) return cudaLaunchKernelEx(&cfg, plan_host_kernel<DA_PLAN_DYNAMIC>, p, h);
  return cudaLaunchKernelEx(&cfg, plan_host_kernel<DA_PLAN_STATIC>, p, h);
}

cudaError_t launch_plan_append(const PlanParams& p, const AppendParams& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1 + (unsigned)min(a.batch, 512), 1, 1);
  cfg.blockDim = dim3(kPlanThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, plan_append_kernel, p, a);
}

}  // namespace da
