// Steps 4 and 5: gather of the routed tokens' original K/V and exact softmax.
//
// HGA technical summary ("Hierarchical Global Attention (HGA)", gist.science
// 2606.30709), "Metodologia -> Meccanismo Core", item 4: once chunks / groups
// are selected, the original token-level K/V are fetched and the output is a
// standard softmax over that bounded, exact token set; no summary value enters
// the output.
//
// The token list of a query at position p (chunk cur) is laid out virtually as
//   [0, a_end)            sink chunks not overlapping the local window
//   [b0*C, p]             local chunks and the causal part of the current one
//   g tokens per group    of every routed group id, in id order
// with b0 = max(0, cur - local) and a_end = min(sink, b0) * C.  Routed groups
// belong to candidate chunks (sink <= c < cur - local), so the three parts never
// overlap and no token is counted twice.
//
// This is the general kernel: any storage type, D in {64, 128}, G <= 16, one
// CTA per (query row, KV head, split).  Decode splits the list (split-K flash
// decoding) and a second kernel merges the partial (o, m, l) by log-sum-exp;
// prefill rows run unsplit and write the output directly.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace hga {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kTile = 32;
constexpr int kGMax = 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TokenList {
  int64_t a_end;   // sink part length (tokens 0 .. a_end-1)
  int64_t b_base;  // first token of the local/current part
  int64_t b_len;   // local/current part length
  int n_groups;    // routed groups kept
  int g;

  __device__ __forceinline__ int64_t total() const {
    return a_end + b_len + static_cast<int64_t>(n_groups) * g;
  }
  __device__ __forceinline__ int64_t token(int64_t v, const int* gl) const {
    if (v < a_end) return v;
    v -= a_end;
    if (v < b_len) return b_base + v;
    v -= b_len;
    return static_cast<int64_t>(gl[v / g]) * g + v % g;
  }
};

// Number of tokens a split covers for the decode launch of p.
__host__ __device__ __forceinline__ int64_t max_tokens(const LayerParams& p) {
  return static_cast<int64_t>(p.sink + p.local + 1) * p.C + static_cast<int64_t>(p.kg) * p.g;
}

int choose_split_tokens(const LayerParams& p, int* nsplit) {
  const int64_t tmax = max_tokens(p);
  if (p.q_len != 1) {
    *nsplit = 1;
    return static_cast<int>(tmax);
  }
  const int64_t items = static_cast<int64_t>(p.B) * p.Hkv;
  const int64_t want = static_cast<int64_t>(device_sm_count()) * 4;  // a few waves
  int64_t per = (tmax * items + want - 1) / want;
  per = ((per + kTile - 1) / kTile) * kTile;
  per = per < 64 ? 64 : (per > 512 ? 512 : per);
  *nsplit = static_cast<int>((tmax + per - 1) / per);
  return static_cast<int>(per);
}

template <typename T, int D, typename TO>
__global__ void __launch_bounds__(kThreads)
attend_kernel(const T* __restrict__ q, const int64_t* __restrict__ pos, const T* __restrict__ k,
              const T* __restrict__ v, const int32_t* __restrict__ group_idx, LayerParams p,
              int nsplit, int split_tokens, TO* __restrict__ out, float* __restrict__ lse,
              float* __restrict__ ws_o, float* __restrict__ ws_ml, unsigned* err) {
  constexpr int DPL = D / 32;        // dims per lane in the score phase
  constexpr int HS = kThreads / D;   // head stride in the PV phase
  __shared__ float s_p[kGMax][kTile];
  __shared__ int64_t s_tok[kTile];
  __shared__ float s_m[kGMax], s_l[kGMax], s_scale[kGMax];
  __shared__ int s_ng;
  extern __shared__ int s_gl[];      // [kg] routed group ids kept

  const int item = blockIdx.x;
  const int split = blockIdx.y;
  const int r = item % p.q_len;
  const int bh = item / p.q_len;
  const int h = bh % p.Hkv, b = bh / p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int d = tid % D;
  pdl_wait();

  const int64_t pb = pos[b];
  const bool ok = valid_position(pb, p, tid == 0 && split == 0 ? err : nullptr);
  const int64_t qpos = pb - p.q_len + 1 + r;
  const int cur = ok ? static_cast<int>(qpos / p.C) : 0;
  const int blk = p.q_len == 1 ? 0 : r / p.C;
  const int b0 = max(0, cur - p.local);

  if (ok) {
    const int32_t* gl = group_idx + (static_cast<size_t>(bh) * p.nblk + blk) * p.kg;
    for (int i = tid; i < p.kg; i += kThreads) s_gl[i] = gl[i];
  }
  if (tid < kGMax) { s_m[tid] = -CUDART_INF_F; s_l[tid] = 0.f; }
  __syncthreads();
  if (tid == 0) {
    int n = 0, prev = -1;
    bool bad = false;
    if (ok) {
      for (int i = 0; i < p.kg; ++i) {
        const int gid = s_gl[i];
        if (gid < 0) continue;
        const int c = gid / p.Ng;
        if (c < p.sink || c >= cur - p.local || gid <= prev) { bad = true; continue; }
        s_gl[n++] = gid;
        prev = gid;
      }
    }
    s_ng = n;
    if (bad && split == 0) flag_error(err, kErrGroupIdx);
  }
  __syncthreads();

  TokenList tl;
  tl.a_end = static_cast<int64_t>(min(p.sink, b0)) * p.C;
  tl.b_base = static_cast<int64_t>(b0) * p.C;
  tl.b_len = ok ? qpos - tl.b_base + 1 : 0;
  tl.n_groups = s_ng;
  tl.g = p.g;
  const int64_t total = ok ? tl.total() : 0;
  const int64_t t_lo = static_cast<int64_t>(split) * split_tokens;
  const int64_t t_hi = min(total, t_lo + split_tokens);

  const size_t kv_base = static_cast<size_t>(bh) * p.n_alloc * D;
  const float qscale = kLog2e * rsqrtf(static_cast<float>(D));
  float qr[kGMax][DPL];
#pragma unroll
  for (int hh = 0; hh < kGMax; ++hh) {
    if (hh < p.G) {
      const T* src = q + ((static_cast<size_t>(b) * p.Hq + h * p.G + hh) * p.q_len + r) * D +
                     lane * DPL;
      if constexpr (DPL == 4) load4(src, qr[hh]); else load2(src, qr[hh]);
#pragma unroll
      for (int u = 0; u < DPL; ++u) qr[hh][u] *= qscale;
    }
  }
  float acc[kGMax];
#pragma unroll
  for (int j = 0; j < kGMax; ++j) acc[j] = 0.f;

  for (int64_t t0 = t_lo; t0 < t_hi; t0 += kTile) {
    const int nt = t_hi - t0 < kTile ? static_cast<int>(t_hi - t0) : kTile;
    if (tid < nt) s_tok[tid] = tl.token(t0 + tid, s_gl);
    __syncthreads();
    // scores (log2 domain): warp per token, lanes over dims
    for (int i = wid; i < nt; i += kWarps) {
      const T* krow = k + kv_base + s_tok[i] * D + lane * DPL;
      float kx[DPL];
      if constexpr (DPL == 4) load4(krow, kx); else load2(krow, kx);
#pragma unroll
      for (int hh = 0; hh < kGMax; ++hh) {
        if (hh < p.G) {
          float s = 0.f;
#pragma unroll
          for (int u = 0; u < DPL; ++u) s += qr[hh][u] * kx[u];
          s = warp_sum(s);
          if (lane == 0) s_p[hh][i] = s;
        }
      }
    }
    __syncthreads();
    // online softmax: warp per head, lane per token
    for (int hh = wid; hh < p.G; hh += kWarps) {
      const float s = lane < nt ? s_p[hh][lane] : -CUDART_INF_F;
      const float m_old = s_m[hh];
      const float m_new = fmaxf(m_old, warp_max(s));
      const float e = lane < nt ? exp2f(s - m_new) : 0.f;
      const float sum = warp_sum(e);
      s_p[hh][lane] = e;
      __syncwarp();
      if (lane == 0) {
        const float sc = m_old == -CUDART_INF_F ? 0.f : exp2f(m_old - m_new);
        s_scale[hh] = sc;
        s_l[hh] = s_l[hh] * sc + sum;
        s_m[hh] = m_new;
      }
    }
    __syncthreads();
    // PV: thread owns dim d of heads tid/D, tid/D + HS, ...
#pragma unroll
    for (int j = 0; j < kGMax; ++j) {
      const int hh = tid / D + j * HS;
      if (hh < p.G) acc[j] *= s_scale[hh];
    }
    for (int i = 0; i < nt; ++i) {
      const float vv = to_f32(v[kv_base + s_tok[i] * D + d]);
#pragma unroll
      for (int j = 0; j < kGMax; ++j) {
        const int hh = tid / D + j * HS;
        if (hh < p.G) acc[j] += s_p[hh][i] * vv;
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int j = 0; j < kGMax; ++j) {
    const int hh = tid / D + j * HS;
    if (hh >= p.G) continue;
    const float m = s_m[hh], l = s_l[hh];
    if (nsplit == 1) {
      const size_t row = (static_cast<size_t>(b) * p.Hq + h * p.G + hh) * p.q_len + r;
      store_out(out + row * D + d, l > 0.f ? acc[j] / l : 0.f);
      if (lse && d == 0) lse[row] = l > 0.f ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
    } else {
      const size_t slot = (static_cast<size_t>(bh) * nsplit + split) * p.G + hh;
      ws_o[slot * D + d] = acc[j];
      if (d == 0) { ws_ml[slot * 2] = m; ws_ml[slot * 2 + 1] = l; }
    }
  }
  pdl_trigger();
}

// Log-sum-exp merge of the split partials of one decode query head.
template <int D, typename TO>
__global__ void __launch_bounds__(D)
combine_kernel(LayerParams p, int nsplit, const float* __restrict__ ws_o,
               const float* __restrict__ ws_ml, TO* __restrict__ out, float* __restrict__ lse) {
  const int bhq = blockIdx.x;
  const int b = bhq / p.Hq, hq = bhq % p.Hq;
  const int h = hq / p.G, hh = hq % p.G;
  const int bh = b * p.Hkv + h;
  const int d = threadIdx.x;
  pdl_wait();
  float m = -CUDART_INF_F;
  for (int s = 0; s < nsplit; ++s) m = fmaxf(m, ws_ml[((static_cast<size_t>(bh) * nsplit + s) * p.G + hh) * 2]);
  float l = 0.f, o = 0.f;
  if (m != -CUDART_INF_F) {
    for (int s = 0; s < nsplit; ++s) {
      const size_t slot = (static_cast<size_t>(bh) * nsplit + s) * p.G + hh;
      const float ms = ws_ml[slot * 2];
      if (ms == -CUDART_INF_F) continue;
      const float w = exp2f(ms - m);
      l += ws_ml[slot * 2 + 1] * w;
      o += ws_o[slot * D + d] * w;
    }
  }
  const size_t row = static_cast<size_t>(b) * p.Hq + hq;  // q_len == 1
  store_out(out + row * D + d, l > 0.f ? o / l : 0.f);
  if (lse && d == 0) lse[row] = l > 0.f ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
  pdl_trigger();
}

}  // namespace

cudaError_t launch_combine(const LayerParams& p, int out_dtype, int nsplit, const float* ws_o,
                           const float* ws_ml, void* out, float* lse, cudaStream_t s) {
  using bf = __nv_bfloat16;
  const dim3 grid(p.B * p.Hq);
  if (p.D == 64)
    return out_dtype == 0
               ? launch_pdl(combine_kernel<64, float>, grid, dim3(64), 0, s, 1, p, nsplit, ws_o,
                            ws_ml, static_cast<float*>(out), lse)
               : launch_pdl(combine_kernel<64, bf>, grid, dim3(64), 0, s, 1, p, nsplit, ws_o,
                            ws_ml, static_cast<bf*>(out), lse);
  return out_dtype == 0
             ? launch_pdl(combine_kernel<128, float>, grid, dim3(128), 0, s, 1, p, nsplit, ws_o,
                          ws_ml, static_cast<float*>(out), lse)
             : launch_pdl(combine_kernel<128, bf>, grid, dim3(128), 0, s, 1, p, nsplit, ws_o,
                          ws_ml, static_cast<bf*>(out), lse);
}

namespace {

template <typename T, int D, typename TO>
cudaError_t launch_attend_t(const LayerParams& p, const void* q, const int64_t* pos, const void* k,
                            const void* v, const int32_t* group_idx, void* out, float* lse,
                            void* ws, unsigned* err, cudaStream_t s) {
  int nsplit = 1;
  const int split_tokens = choose_split_tokens(p, &nsplit);
  float* ws_o = static_cast<float*>(ws);
  float* ws_ml = ws_o ? ws_o + static_cast<size_t>(p.B) * p.Hkv * nsplit * p.G * D : nullptr;
  const size_t smem = static_cast<size_t>(p.kg) * sizeof(int);
  cudaError_t e = ensure_smem<attend_kernel<T, D, TO>>(smem);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(static_cast<int64_t>(p.B) * p.Hkv * p.q_len), nsplit);
  e = launch_pdl(attend_kernel<T, D, TO>, grid, dim3(kThreads), smem, s, 1,
                 static_cast<const T*>(q), pos, static_cast<const T*>(k),
                 static_cast<const T*>(v), group_idx, p, nsplit, split_tokens,
                 static_cast<TO*>(out), lse, ws_o, ws_ml, err);
  if (e != cudaSuccess || nsplit == 1) return e;
  return launch_combine(p, std::is_same<TO, float>::value ? 0 : 1, nsplit, ws_o, ws_ml, out, lse, s);
}

template <typename T, typename TO>
cudaError_t launch_attend_d(const LayerParams& p, const void* q, const int64_t* pos, const void* k,
                            const void* v, const int32_t* gi, void* out, float* lse, void* ws,
                            unsigned* err, cudaStream_t s) {
  return p.D == 64 ? launch_attend_t<T, 64, TO>(p, q, pos, k, v, gi, out, lse, ws, err, s)
                   : launch_attend_t<T, 128, TO>(p, q, pos, k, v, gi, out, lse, ws, err, s);
}

}  // namespace

static bool use_decode_fast(const LayerParams& p, int dtype) {
  return decode_fast_path(p, dtype) &&
         static_cast<int64_t>(p.B) * p.Hkv * p.n_alloc < (static_cast<int64_t>(1) << 31);
}

size_t attend_workspace_bytes(const LayerParams& p, int dtype) {
  if (use_decode_fast(p, dtype)) return 0;  // partials merge inside a thread-block cluster
  int nsplit = 1;
  choose_split_tokens(p, &nsplit);
  if (nsplit == 1) return 0;
  return static_cast<size_t>(p.B) * p.Hkv * nsplit * p.G * (p.D + 2) * sizeof(float);
}

cudaError_t launch_attend(const LayerParams& p, int dtype, int out_dtype, const void* q,
                          const int64_t* pos, const void* k, const void* v,
                          const int32_t* group_idx, void* out, float* lse, void* ws,
                          unsigned* err, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (use_decode_fast(p, dtype))
    return launch_attend_decode_bf16(p, out_dtype, q, pos, k, v, group_idx, out, lse, err, 0, s);
  if (prefill_tc_path(p, dtype))
    return launch_attend_prefill_bf16(p, out_dtype, q, pos, k, v, group_idx, out, lse, err, s);
  if (dtype == 0)
    return out_dtype == 0 ? launch_attend_d<float, float>(p, q, pos, k, v, group_idx, out, lse, ws, err, s)
                          : launch_attend_d<float, bf>(p, q, pos, k, v, group_idx, out, lse, ws, err, s);
  return out_dtype == 0 ? launch_attend_d<bf, float>(p, q, pos, k, v, group_idx, out, lse, ws, err, s)
                        : launch_attend_d<bf, bf>(p, q, pos, k, v, group_idx, out, lse, ws, err, s);
}

}  // namespace hga
