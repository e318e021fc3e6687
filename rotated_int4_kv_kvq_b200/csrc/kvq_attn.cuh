// kvq_attn.cuh -- decode attention that reads the int4 cache directly.
//
// "Day 9 - Quantization: Shrink the Bytes Themselves", section "Decode into
// HBM, or Decode into Registers": the dequantization runs inside the kernel
// that consumes it, so only int4 codes and scales cross HBM and the decoded
// K/V exist in registers only.  With the rotation this goes one step
// further: R is orthonormal, so <q, D R^T y_K> = <R D q, y_K> and
// sum_t p_t D R^T y_V,t = D R^T (sum_t p_t y_V,t).  The kernel rotates each
// query once, scores every token against y_K = s q_codes in the rotated
// domain, accumulates sum p_t y_V,t there, and rotates the result back once
// per query: no per-token FFT.
//
// Layout of the work: one thread-block cluster of C blocks per KV head; each
// block takes a contiguous share of the tokens and its 8 warps take blocks
// of TB = 32 / NQ tokens in turn.  Inside a warp, lane l owns the W = d/32
// rotated coordinates of chunk k2 (the one-warp-per-vector layout of
// kvq_wide.cuh), so a token's codes are one coalesced load per lane.  The
// NQ x TB partial dot products of a token block are summed across lanes by
// one reduce-scatter (31 shuffles leave lane qi*TB + tb holding the score of
// query qi and token tb), then an online softmax (base 2) rescales the
// accumulators once per block.  Warps, then blocks, merge their (max, sum,
// accumulator) triples through shared memory and distributed shared memory
// of the cluster: no global scratch.
#pragma once

#include <cooperative_groups.h>

#include "kvq_wide.cuh"

namespace kvq {

constexpr int kAttnWarps = 8;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr int kAttnChunk = 32;   // tokens per staged chunk of a warp
constexpr int kAttnStages = 2;   // chunks in flight per warp
constexpr int kAttnMaxCluster = 16;  // blocks per KV head at most

// Asynchronous global -> shared copies (cp.async); `bytes` < size zero-fills
// the rest and 0 reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Shared-memory bytes of one staged chunk (K and V codes, K and V scales;
// scales sized for the smallest group, 32).
template <int D>
constexpr int attn_chunk_bytes() {
  return 2 * kAttnChunk * (D / 2) + 2 * kAttnChunk * (D / 32) * 4;
}

struct AttnArgs {
  const uint16_t* q;         // [n_kv][nq][d] fp16
  const uint8_t* k_packed;   // [n_kv][cap][d/2]
  const float* k_scales;     // [n_kv][cap][d/g]
  const uint8_t* v_packed;
  const float* v_scales;
  uint16_t* out;             // [n_kv][nq][d] fp16
  const int8_t* signs;
  int64_t cap, len;
  int nq;                    // queries per KV head (<= NQ; the rest are padding)
  int group;
  float qscale;              // sm_scale * KAPPA * log2(e)
};

// Per-warp (or per-block) partial state of one query: running max m (base 2),
// sum l, and the lane's W accumulated rotated coordinates.
template <int D, int NQ>
struct AttnPartial {
  static constexpr int W = D / 32;
  // shared-memory floats per partial: m, l for each query, then NQ x D acc
  static constexpr int FLOATS = 2 * NQ + NQ * D;
};

// Sum of 32 values per lane across the warp, scattered: lane l ends with
// the total of index l.
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = lane & o;
#pragma unroll
    for (int j = 0; j < o; ++j) {
      const float send = upper ? v[j] : v[j + o];
      const float keep = upper ? v[j + o] : v[j];
      v[j] = keep + __shfl_xor_sync(kFull, send, o);
    }
  }
  return v[0];
}

// The lane's code bytes (W/2) of a staged row.
template <int D>
__device__ __forceinline__ uint32_t attn_lds_code(uint32_t row, int k2) {
  constexpr int QB = D / 64;  // code bytes per lane: W / 2
  if constexpr (QB == 4) {
    return lds32(row + uint32_t(k2 * 4));
  } else {
    uint32_t v;
    if constexpr (QB == 2) {
      asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(row + uint32_t(k2 * 2)) : "memory");
    } else {
      asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(row + uint32_t(k2)) : "memory");
    }
    return v;
  }
}

// The lane's W codes as W/2 pairs of floats.
template <int C>
__device__ __forceinline__ void attn_unpack(uint32_t code, f2 (&c)[C]) {
  f2 q[4];
  unpack8(code, q);
  const f2 magic = mk2(kUnpackMagic, kUnpackMagic);
#pragma unroll
  for (int j = 0; j < C; ++j) c[j] = sub2(q[j], magic);
}

// Merges the per-warp partials in shared memory (slot w of s_part: m and l
// of every query, then the NQ x D accumulated rotated coordinates, written
// before the call) across the block and the cluster: the block's triple goes
// to its slot 0, the cluster's blocks merge into slot 1 of block 0, a slice
// each, and block 0 rotates every query's result back and stores it.
template <int D, int ROT, int NQ>
__device__ __forceinline__ void attn_merge_store(const AttnArgs& a, float* s_part,
                                                 cooperative_groups::cluster_group& cluster,
                                                 int rank, int nblk, int64_t head, int warp,
                                                 int lane, const WideLane<D, ROT>& L) {
  using P = Wide<D, ROT>;
  constexpr int W = P::W, C = P::C;
  using AP = AttnPartial<D, NQ>;
  const int k2 = L.k2;
  float* stage = s_part + kAttnWarps * AP::FLOATS;
  __syncthreads();
  // per query, the weight f_w = 2^(m_w - max_w m_w) of every warp's partial,
  // formed once (warp qi for query qi, lane w for warp w's partial, max and
  // sum by shuffles); then thread i merges element i of every (query,
  // coordinate) and leaves the block's triple in warp slot 0
  __shared__ float s_bw[kAttnWarps * NQ];
  static_assert(NQ <= kAttnWarps && kAttnWarps <= 32, "one warp per query, a lane per warp");
  if (warp < NQ) {
    const int qi = warp;
    const bool has = lane < kAttnWarps;
    const float mw = has ? s_part[lane * AP::FLOATS + 2 * qi] : -INFINITY;
    const float lw = has ? s_part[lane * AP::FLOATS + 2 * qi + 1] : 0.0f;
    float mm = mw;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(kFull, mm, o));
    const float f = mw == -INFINITY ? 0.0f : exp2f(mw - mm);
    float ls = f * lw;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(kFull, ls, o);
    if (has) s_bw[lane * NQ + qi] = f;
    if (lane == 0) {  // m, l of every slot are still being read: stage them
      stage[2 * qi] = mm;
      stage[2 * qi + 1] = ls;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < NQ * D; e += kAttnThreads) {
    const int qi = e / D;
    float accv = 0.0f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w)
      accv += s_bw[w * NQ + qi] * s_part[w * AP::FLOATS + 2 * NQ + e];
    s_part[2 * NQ + e] = accv;  // slot 0 (warp 0's region): read only by this thread
  }
  __syncthreads();
  if (threadIdx.x < 2 * NQ) s_part[threadIdx.x] = stage[threadIdx.x];
  cluster.sync();  // every block's triple is in its slot 0

  // ---- the cluster's blocks merge into slot 1 of block 0, a slice each ----
  // weights of every block's triple per query: f_b / sum_b f_b l_b with
  // f_b = 2^(m_b - max_b m_b); each block reads the (m, l) pairs once, one
  // remote read per thread, and forms the weights in its own shared memory
  __shared__ float s_w[kAttnMaxCluster * NQ];
  __shared__ float s_l[kAttnMaxCluster * NQ];
  for (int i = threadIdx.x; i < nblk * NQ; i += kAttnThreads) {
    const float* src = cluster.map_shared_rank(s_part, i / NQ);
    s_w[i] = src[2 * (i % NQ)];
    s_l[i] = src[2 * (i % NQ) + 1];
  }
  __syncthreads();
  static_assert(kAttnMaxCluster <= 32, "a lane per block of the cluster");
  if (warp < NQ) {  // warp qi: lane b forms block b's weight, max and sum by shuffles
    const int qi = warp;
    const bool has = lane < nblk;
    const float mb = has ? s_w[lane * NQ + qi] : -INFINITY;
    const float lb = has ? s_l[lane * NQ + qi] : 0.0f;
    float mm = mb;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(kFull, mm, o));
    const float f = mb == -INFINITY ? 0.0f : exp2f(mb - mm);
    float ls = f * lb;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(kFull, ls, o);
    if (has) s_w[lane * NQ + qi] = f * (1.0f / ls);
  }
  __syncthreads();
  {
    float* fin = cluster.map_shared_rank(s_part, 0) + AP::FLOATS;
    constexpr int NE = NQ * D;
    const int per = (NE + nblk - 1) / nblk;
    const int e_end = (rank + 1) * per < NE ? (rank + 1) * per : NE;
    for (int e = rank * per + threadIdx.x; e < e_end; e += kAttnThreads) {
      const int qi = e / D;
      float accv = 0.0f;
#pragma unroll 4
      for (int b = 0; b < nblk; ++b)
        accv += s_w[b * NQ + qi] * cluster.map_shared_rank(s_part, b)[2 * NQ + e];
      fin[2 * NQ + e] = accv;
    }
  }
  cluster.sync();  // block 0's slot 1 is complete; remote reads done, others may exit
  if (rank == 0 && warp < a.nq) {
    const int qi = warp;
    const float* fin = s_part + AP::FLOATS + 2 * NQ + qi * D;
    float Y[W];
#pragma unroll
    for (int w = 0; w < W; ++w) Y[w] = fin[k2 * W + w] * P::KAPPA;
    uint32_t xo[C];
    wide_rotate_inv<D, ROT>(Y, L, xo);
    wide_store_words<D, ROT>(a.out + (head * a.nq + qi) * D, L, xo);
  }
}

template <int D, int ROT, int NQ>
__global__ void __launch_bounds__(kAttnThreads, 1) kvq_attn_kernel(const AttnArgs a) {
  namespace cg = cooperative_groups;
  using P = Wide<D, ROT>;
  constexpr int W = P::W, C = P::C;
  constexpr int TB = 32 / NQ;  // tokens per block
  using AP = AttnPartial<D, NQ>;
  extern __shared__ __align__(16) float s_part[];  // staging rings, then merge slots

  pdl_wait();  // no global access before the previous kernel completes
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int nblk = int(cluster.num_blocks());
  const int64_t head = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WideLane<D, ROT> L;
  L.init(a.signs, lane);
  const int k2 = L.k2;
  const int grp = (k2 * W) / a.group;
  const int ng = D / a.group;

  // this block's tokens, then this warp's contiguous share (whole token
  // blocks of TB)
  const int64_t per = (a.len + nblk - 1) / nblk;
  const int64_t t_begin = int64_t(rank) * per;
  const int64_t t_end = t_begin + per < a.len ? t_begin + per : a.len;
  const int64_t per_w = ((t_end - t_begin + kAttnWarps - 1) / kAttnWarps + TB - 1) / TB * TB;
  const int64_t w_begin = t_begin + int64_t(warp) * per_w;
  const int64_t w_end = w_begin + per_w < t_end ? w_begin + per_w : t_end;
  const int64_t n_w = w_end > w_begin ? w_end - w_begin : 0;
  const uint8_t* kbase = a.k_packed + head * a.cap * (D / 2);
  const uint8_t* vbase = a.v_packed + head * a.cap * (D / 2);
  const float* ksc = a.k_scales + head * a.cap * ng;
  const float* vsc = a.v_scales + head * a.cap * ng;

  // staging ring of this warp: [stage][K codes | V codes | K scales | V scales]
  constexpr int QROW = D / 2;
  constexpr int CB = attn_chunk_bytes<D>();
  const uint32_t ring = smem_u32(s_part) + uint32_t(warp * kAttnStages * CB);
  const int nchunk = int((n_w + kAttnChunk - 1) / kAttnChunk);
  auto issue = [&](int c) {
    if (c < nchunk) {
      const uint32_t st = ring + uint32_t((c % kAttnStages) * CB);
      const int64_t r0 = w_begin + int64_t(c) * kAttnChunk;
      const int rows = int(w_end - r0 < kAttnChunk ? w_end - r0 : kAttnChunk);
      constexpr int PIECES = kAttnChunk * QROW / 16;  // 16-byte pieces per code tile
#pragma unroll
      for (int i = lane; i < PIECES; i += 32) {
        const int row = i / (QROW / 16);
        const bool ok = row < rows;
        const int64_t off = ok ? (r0 + row) * QROW + (i % (QROW / 16)) * 16 : r0 * QROW;
        cp_async16(st + uint32_t(i * 16), kbase + off, ok ? 16 : 0);
        cp_async16(st + uint32_t(kAttnChunk * QROW + i * 16), vbase + off, ok ? 16 : 0);
      }
      const uint32_t sk = st + uint32_t(2 * kAttnChunk * QROW);
      const uint32_t sv = sk + uint32_t(kAttnChunk * (D / 32) * 4);
      for (int i = lane; i < kAttnChunk * ng; i += 32) {
        const int row = i / ng;
        const bool ok = row < rows;
        const int64_t off = ok ? (r0 + row) * ng + i % ng : r0 * ng;
        cp_async4(sk + uint32_t(i * 4), ksc + off, ok ? 4 : 0);
        cp_async4(sv + uint32_t(i * 4), vsc + off, ok ? 4 : 0);
      }
    }
    cp_async_commit();  // possibly empty: keeps the group count uniform
  };
#pragma unroll
  for (int c = 0; c < kAttnStages; ++c) issue(c);

  // rotated queries, pre-scaled (score = <qr, y_K> in log2 units): warp w
  // rotates query w into shared memory, then every warp loads all of them
  float* s_q = s_part + kAttnWarps * kAttnStages * (attn_chunk_bytes<D>() / 4);
  for (int qi = warp; qi < NQ; qi += kAttnWarps) {
    uint32_t xw[C];
    if (qi < a.nq) {
      wide_load_words<D, ROT>(a.q + (head * a.nq + qi) * D, L, xw);
    } else {
#pragma unroll
      for (int j = 0; j < C; ++j) xw[j] = 0u;
    }
    float Y[W];
    wide_rotate_fwd<D, ROT>(xw, L, Y);
#pragma unroll
    for (int w = 0; w < W; ++w) s_q[qi * D + k2 * W + w] = Y[w] * a.qscale;
  }
  __syncthreads();
  f2 qr[NQ][C];
#pragma unroll
  for (int qi = 0; qi < NQ; ++qi)
#pragma unroll
    for (int j = 0; j < C; ++j)
      qr[qi][j] = mk2(s_q[qi * D + k2 * W + 2 * j], s_q[qi * D + k2 * W + 2 * j + 1]);

  float m = -INFINITY, l = 0.0f;  // of query lane / TB
  f2 acc[NQ][C];
#pragma unroll
  for (int qi = 0; qi < NQ; ++qi)
#pragma unroll
    for (int j = 0; j < C; ++j) acc[qi][j] = mk2(0.0f, 0.0f);

  for (int c = 0; c < nchunk; ++c) {
    cp_async_wait<kAttnStages - 1>();
    __syncwarp();
    const uint32_t st = ring + uint32_t((c % kAttnStages) * CB);
    const uint32_t skc = st, svc = st + uint32_t(kAttnChunk * QROW);
    const uint32_t sks = st + uint32_t(2 * kAttnChunk * QROW);
    const uint32_t svs = sks + uint32_t(kAttnChunk * (D / 32) * 4);
    const int rows = int(w_end - (w_begin + int64_t(c) * kAttnChunk) < kAttnChunk
                             ? w_end - (w_begin + int64_t(c) * kAttnChunk)
                             : kAttnChunk);
    // scores of the whole chunk first (independent per token block), then
    // one softmax update and the V accumulation
    constexpr int NB = kAttnChunk / TB;  // token blocks per chunk
    float score[NB];
#pragma unroll
    for (int bi = 0; bi < NB; ++bi) score[bi] = -INFINITY;
#pragma unroll 1
    for (int bi = 0; bi < NB; ++bi) {
      if (bi * TB >= rows) break;
      float part[32];
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) {
        const int r = bi * TB + tb;  // rows >= `rows` are zero-filled: code 0, scale 0
        const uint32_t code = attn_lds_code<D>(skc + uint32_t(r * QROW), k2);
        const float sk = __uint_as_float(lds32(sks + uint32_t((r * ng + grp) * 4)));
        f2 cc[C];
        attn_unpack<C>(code, cc);
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) {
          f2 s2 = mul2(qr[qi][0], cc[0]);
#pragma unroll
          for (int j = 1; j < C; ++j) s2 = fma2(qr[qi][j], cc[j], s2);
          part[qi * TB + tb] = (lo2(s2) + hi2(s2)) * sk;
        }
      }
      float sc = reduce_scatter32(part, lane);  // query lane / TB, token bi*TB + lane % TB
      if (bi * TB + (lane % TB) >= rows) sc = -INFINITY;
#pragma unroll
      for (int k = 0; k < NB; ++k)
        if (k == bi) score[k] = sc;
    }
    float bmax = score[0];
#pragma unroll
    for (int bi = 1; bi < NB; ++bi) bmax = fmaxf(bmax, score[bi]);
#pragma unroll
    for (int o = TB / 2; o >= 1; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, o));
    const float m_new = fmaxf(m, bmax);  // finite: the chunk holds a valid token
    const float corr = exp2f(m - m_new);
    float p[NB];
    float psum = 0.0f;
#pragma unroll
    for (int bi = 0; bi < NB; ++bi) {
      p[bi] = exp2f(score[bi] - m_new);
      psum += p[bi];
    }
#pragma unroll
    for (int o = TB / 2; o >= 1; o >>= 1) psum += __shfl_xor_sync(kFull, psum, o);
    l = l * corr + psum;
    m = m_new;
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
      const float cq = __shfl_sync(kFull, corr, qi * TB);
      const f2 c2 = mk2(cq, cq);
#pragma unroll
      for (int j = 0; j < C; ++j) acc[qi][j] = mul2(acc[qi][j], c2);
    }
#pragma unroll 1
    for (int bi = 0; bi < NB; ++bi) {
      if (bi * TB >= rows) break;
      float pb = p[0];
#pragma unroll
      for (int k = 1; k < NB; ++k)
        if (k == bi) pb = p[k];
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) {
        const int r = bi * TB + tb;
        const uint32_t code = attn_lds_code<D>(svc + uint32_t(r * QROW), k2);
        const float sv = __uint_as_float(lds32(svs + uint32_t((r * ng + grp) * 4)));
        f2 cc[C];
        attn_unpack<C>(code, cc);
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) {
          const float w = __shfl_sync(kFull, pb, qi * TB + tb) * sv;
          const f2 w2 = mk2(w, w);
#pragma unroll
          for (int j = 0; j < C; ++j) acc[qi][j] = fma2(w2, cc[j], acc[qi][j]);
        }
      }
    }
    __syncwarp();  // the stage is consumed before it is refilled
    issue(c + kAttnStages);
  }
  cp_async_wait<0>();
  pdl_release();
  __syncthreads();  // the staging rings become the merge area

  // ---- this warp's partial into its merge slot ----
  float* mine = s_part + warp * AP::FLOATS;
  if (lane % TB == 0) {
    mine[2 * (lane / TB)] = m;
    mine[2 * (lane / TB) + 1] = l;
  }
#pragma unroll
  for (int qi = 0; qi < NQ; ++qi)
#pragma unroll
    for (int j = 0; j < C; ++j) {
      float* dst = mine + 2 * NQ + qi * D + k2 * W + 2 * j;
      dst[0] = lo2(acc[qi][j]);
      dst[1] = hi2(acc[qi][j]);
    }
  attn_merge_store<D, ROT, NQ>(a, s_part, cluster, rank, nblk, head, warp, lane, L);
}

// Dynamic shared memory of kvq_attn_kernel.
template <int D, int NQ>
constexpr int attn_smem_bytes() {
  constexpr int merge = (kAttnWarps * AttnPartial<D, NQ>::FLOATS + 2 * NQ) * 4;
  constexpr int staging = kAttnWarps * kAttnStages * attn_chunk_bytes<D>() + NQ * D * 4;
  return merge > staging ? merge : staging;
}

}  // namespace kvq
