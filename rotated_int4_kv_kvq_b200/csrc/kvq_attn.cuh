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

// Iterations of a warp's tokens in flight in the lane-pair kernel (cp.async
// into shared memory; 0: plain loads into registers, two tokens ahead).
#ifndef KVQ_ATTN_PAIR_STAGES
#define KVQ_ATTN_PAIR_STAGES 3
#endif
// Unpack codes in the lane-pair kernel through fp16 and mixed-precision
// multiply-adds (1) or byte permutes into offset floats (0).
#ifndef KVQ_ATTN_MIXED_UNPACK
#define KVQ_ATTN_MIXED_UNPACK 1
#endif

// Lazy online softmax (the lane-pair and tensor-core kernels): a running
// reference maximum m moves only when a new score exceeds it by more than
// kAttnSlack (log2 units), so weights 2^(s - m) stay below 2^kAttnSlack and
// the accumulators are rescaled only then; the warp, block and cluster
// merges take any reference m with its (l, o).
constexpr float kAttnSlack = 8.0f;

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
  int qgroups;               // tensor-core kernel: blocks of 4 queries per KV head
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
                                                 int lane, const WideLane<D, ROT>& L,
                                                 int q0 = 0, int qn = -1) {
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
  if (rank == 0 && warp < (qn < 0 ? a.nq : qn)) {  // queries q0 .. of the KV head
    const int qi = warp;
    const float* fin = s_part + AP::FLOATS + 2 * NQ + qi * D;
    float Y[W];
#pragma unroll
    for (int w = 0; w < W; ++w) Y[w] = fin[k2 * W + w] * P::KAPPA;
    uint32_t xo[C];
    wide_rotate_inv<D, ROT>(Y, L, xo);
    wide_store_words<D, ROT>(a.out + (head * a.nq + q0 + qi) * D, L, xo);
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
  // whole chunks: every lane copies fixed pieces from running source
  // pointers (piece i = lane + 32k of the code tile is row i / PR, 16-byte
  // column i % PR), and the chunk's scales as one contiguous run (16-byte
  // pieces where both scale bases allow it); the last, partial chunk takes
  // the checked path
  constexpr int PR = QROW / 16;
  const uint8_t* kcur = kbase + (w_begin + lane / PR) * QROW + (lane % PR) * 16;
  const uint8_t* vcur = vbase + (w_begin + lane / PR) * QROW + (lane % PR) * 16;
  const float* kscur = ksc + w_begin * ng;
  const float* vscur = vsc + w_begin * ng;
  const bool sc16 =
      ((reinterpret_cast<uintptr_t>(kscur) | reinterpret_cast<uintptr_t>(vscur)) & 15u) == 0;
  auto issue = [&](int c) {  // called for c = 0, 1, 2, ... in order
    if (c < nchunk) {
      const uint32_t st = ring + uint32_t((c % kAttnStages) * CB);
      const int64_t r0 = w_begin + int64_t(c) * kAttnChunk;
      const int rows = int(w_end - r0 < kAttnChunk ? w_end - r0 : kAttnChunk);
      constexpr int PIECES = kAttnChunk * QROW / 16;  // 16-byte pieces per code tile
      const uint32_t sk = st + uint32_t(2 * kAttnChunk * QROW);
      const uint32_t sv = sk + uint32_t(kAttnChunk * (D / 32) * 4);
      if (rows == kAttnChunk) {
#pragma unroll
        for (int k = 0; k < PIECES / 32; ++k) {
          cp_async16(st + uint32_t((lane + 32 * k) * 16), kcur + k * 512, 16);
          cp_async16(st + uint32_t(kAttnChunk * QROW + (lane + 32 * k) * 16), vcur + k * 512, 16);
        }
        if (sc16) {
          for (int i = lane; i < 8 * ng; i += 32) {  // 32 ng floats in 16-byte pieces
            cp_async16(sk + uint32_t(i * 16), kscur + 4 * i, 16);
            cp_async16(sv + uint32_t(i * 16), vscur + 4 * i, 16);
          }
        } else {
          for (int i = lane; i < kAttnChunk * ng; i += 32) {
            cp_async4(sk + uint32_t(i * 4), kscur + i, 4);
            cp_async4(sv + uint32_t(i * 4), vscur + i, 4);
          }
        }
        kcur += kAttnChunk * QROW;
        vcur += kAttnChunk * QROW;
        kscur += kAttnChunk * ng;
        vscur += kAttnChunk * ng;
        cp_async_commit();
        return;
      }
#pragma unroll
      for (int i = lane; i < PIECES; i += 32) {
        const int row = i / (QROW / 16);
        const bool ok = row < rows;
        const int64_t off = ok ? (r0 + row) * QROW + (i % (QROW / 16)) * 16 : r0 * QROW;
        cp_async16(st + uint32_t(i * 16), kbase + off, ok ? 16 : 0);
        cp_async16(st + uint32_t(kAttnChunk * QROW + i * 16), vbase + off, ok ? 16 : 0);
      }
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

// Dynamic shared memory of kvq_attn_pair_kernel: the merge slots (which also
// hold the rotated query before the token loop), then the warps' stages.
template <int D>
constexpr int attn_pair_merge_bytes() {
  constexpr int merge = (kAttnWarps * AttnPartial<D, 1>::FLOATS + 2) * 4;
  return ((merge > D * 4 ? merge : D * 4) + 15) / 16 * 16;
}
template <int D>
constexpr int attn_pair_smem_bytes() {
  return attn_pair_merge_bytes<D>() +
         kAttnWarps * KVQ_ATTN_PAIR_STAGES * (2 * 32 * (D / 2) + 32 * 16);
}

// Decode attention at d = 64 with one query per KV head (multi-head caches
// such as SmolLM2's): a pair of lanes per token instead of a warp.  Lane h
// of a pair holds rotated coordinates [32h, 32h + 32) of the query; for each
// of its tokens it reads that half's 16 code bytes and scale of K and of V
// with one 128-bit and one 32-bit load each (consecutive pairs read
// consecutive rows), forms its partial dot product, and the pair adds the two
// halves with one shuffle.  A pair takes two tokens per iteration, 128 rows
// apart, with all eight loads issued before either is used.  Each lane keeps
// its own online softmax (base 2, one update per two tokens) and
// accumulator.  After the loop the 16 pairs of a warp merge by shuffles
// (a reduce-scatter leaves each lane two coordinates), and the block and the
// cluster merge as in kvq_attn_kernel.  Per token a warp issues about a
// third of the instructions of the warp-per-token layout, whose lanes hold
// only two coordinates each at d = 64.
template <int D, int ROT>
__global__ void __launch_bounds__(kAttnThreads, 2) kvq_attn_pair_kernel(const AttnArgs a) {
  static_assert(D == 64, "a lane pair per token: 32 coordinates per lane");
  namespace cg = cooperative_groups;
  constexpr int NQ = 1;
  using P = Wide<D, ROT>;
  constexpr int W = P::W, C = P::C;
  constexpr int HC = D / 2;   // coordinates per lane
  constexpr int NP = HC / 2;  // f2 pairs per lane
  constexpr int QB = HC / 2;  // code bytes per lane and token
  [[maybe_unused]] constexpr int kPairs = kAttnThreads / 2;
  using AP = AttnPartial<D, NQ>;
  extern __shared__ __align__(16) float s_part[];

  pdl_wait();  // no global access before the previous kernel completes
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int nblk = int(cluster.num_blocks());
  const int64_t head = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = lane & 1;
  const int ng = D / a.group;      // scales per token (1 or 2)
  const int sh = ng == 2 ? h : 0;  // the scale of this lane's half

  // this block's tokens
  const int64_t per = (a.len + nblk - 1) / nblk;
  const int64_t t_begin = int64_t(rank) * per;
  const int64_t t_end = t_begin + per < a.len ? t_begin + per : a.len;
  const uint32_t n_tok = uint32_t(t_end > t_begin ? t_end - t_begin : 0);
  const uint32_t pmask = 3u << (lane & 30);
#if KVQ_ATTN_PAIR_STAGES > 0
  // Iteration i of warp w covers tokens ob + [0, 32) of the block's range,
  // ob = 256 i + 32 w; pair pp = lane / 2 takes ob + pp and ob + 16 + pp.
  // Each lane copies its own halves of the two tokens' K and V codes and
  // their scales into a stage of its warp (cp.async, KVQ_ATTN_PAIR_STAGES
  // stages) and reads back only what it copied, so completion is per lane.
  constexpr int S = KVQ_ATTN_PAIR_STAGES;
  constexpr int CB = 32 * (D / 2);         // code bytes of 32 tokens (K or V)
  constexpr int STAGE = 2 * CB + 32 * 16;  // then (sk0, sv0, sk1, sv1) per lane
  const int64_t row0 = head * a.cap + t_begin;
  const uint8_t* kb = a.k_packed + row0 * (D / 2) + QB * h;
  const uint8_t* vb = a.v_packed + row0 * (D / 2) + QB * h;
  const float* ks = a.k_scales + row0 * ng + sh;
  const float* vs = a.v_scales + row0 * ng + sh;
  const int pp = lane >> 1;
  const uint32_t stages =
      smem_u32(s_part) + uint32_t(attn_pair_merge_bytes<D>() + warp * S * STAGE);
  auto issue = [&](uint32_t ob, int s) {
    const uint32_t st = stages + uint32_t(s * STAGE);
    if (ob + 32u <= n_tok) {  // the warp's 32 tokens all in range: no clamps
      const size_t r = size_t(ob) + uint32_t(pp);
      const uint8_t* kp = kb + r * (D / 2);
      const uint8_t* vp = vb + r * (D / 2);
      const float* ksp = ks + r * ng;
      const float* vsp = vs + r * ng;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        cp_async16(st + uint32_t(16 * (32 * j + lane)), kp + 16 * j * (D / 2), 16);
        cp_async16(st + uint32_t(CB + 16 * (32 * j + lane)), vp + 16 * j * (D / 2), 16);
        cp_async4(st + uint32_t(2 * CB + 16 * lane + 8 * j), ksp + 16 * j * ng, 4);
        cp_async4(st + uint32_t(2 * CB + 16 * lane + 8 * j + 4), vsp + 16 * j * ng, 4);
      }
    } else if (ob < n_tok) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t o = ob + 16u * j + uint32_t(pp);
        const uint32_t r = o < n_tok ? o : ob;  // out of range: zero fill from a valid row
        const int n16 = o < n_tok ? 16 : 0, n4 = o < n_tok ? 4 : 0;
        cp_async16(st + uint32_t(16 * (32 * j + lane)), kb + size_t(r) * (D / 2), n16);
        cp_async16(st + uint32_t(CB + 16 * (32 * j + lane)), vb + size_t(r) * (D / 2), n16);
        cp_async4(st + uint32_t(2 * CB + 16 * lane + 8 * j), ks + size_t(r) * ng, n4);
        cp_async4(st + uint32_t(2 * CB + 16 * lane + 8 * j + 4), vs + size_t(r) * ng, n4);
      }
    }
    cp_async_commit();  // one group per iteration, empty past the range
  };
#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(uint32_t(32 * warp + 256 * s), s);
#else
  const uint8_t* kb = a.k_packed + head * a.cap * (D / 2) + QB * h;
  const uint8_t* vb = a.v_packed + head * a.cap * (D / 2) + QB * h;
  const float* ks = a.k_scales + head * a.cap * ng + sh;
  const float* vs = a.v_scales + head * a.cap * ng + sh;
#endif

  // the rotated, pre-scaled query: warp 0 rotates it into shared memory,
  // every lane takes its half
  if (warp == 0) {
    WideLane<D, ROT> L;  // (set up again for the merge: not live through the loop)
    L.init(a.signs, lane);
    uint32_t xw[C];
    wide_load_words<D, ROT>(a.q + head * D, L, xw);
    float Y[W];
    wide_rotate_fwd<D, ROT>(xw, L, Y);
#pragma unroll
    for (int w = 0; w < W; ++w) s_part[L.k2 * W + w] = Y[w] * a.qscale;
  }
  __syncthreads();
  f2 qr[NP];
#pragma unroll
  for (int j = 0; j < NP; ++j) qr[j] = mk2(s_part[HC * h + 2 * j], s_part[HC * h + 2 * j + 1]);
  __syncthreads();  // the query slots become merge slots

  [[maybe_unused]] const f2 magic = mk2(kUnpackMagic, kUnpackMagic);
  float m = -INFINITY, l = 0.0f;
  f2 acc[NP];
#pragma unroll
  for (int j = 0; j < NP; ++j) acc[j] = mk2(0.0f, 0.0f);
  // half of the K dot product of one token (times its scale)
  auto kdot = [&](const uint4& kc, float sk) {
    const uint32_t kw[4] = {kc.x, kc.y, kc.z, kc.w};
    f2 d2 = mk2(0.0f, 0.0f);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      f2 c[4];
#if KVQ_ATTN_MIXED_UNPACK
      unpack8_signed(kw[w], c);
#pragma unroll
      for (int i = 0; i < 4; ++i) d2 = fma2(qr[4 * w + i], c[i], d2);
#else
      unpack8(kw[w], c);
#pragma unroll
      for (int i = 0; i < 4; ++i) d2 = fma2(qr[4 * w + i], sub2(c[i], magic), d2);
#endif
    }
    return (lo2(d2) + hi2(d2)) * sk;
  };
  auto vacc = [&](const uint4& vc, float wv) {
    const uint32_t vw[4] = {vc.x, vc.y, vc.z, vc.w};
    const f2 w2 = mk2(wv, wv);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      f2 c[4];
#if KVQ_ATTN_MIXED_UNPACK
      unpack8_signed(vw[w], c);
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[4 * w + i] = fma2(w2, c[i], acc[4 * w + i]);
#else
      unpack8(vw[w], c);
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[4 * w + i] = fma2(w2, sub2(c[i], magic), acc[4 * w + i]);
#endif
    }
  };
  // one online-softmax update for two scored tokens (s1 = -inf: no second)
  auto update = [&](float s0, float s1, const uint4& vc0, float sv0, const uint4& vc1, float sv1) {
    const float mx = fmaxf(s0, s1);
    if (mx > m + kAttnSlack) {  // the reference moves: rescale (m = -inf: zeros)
      const float corr = exp2f(m - mx);
      const f2 c2 = mk2(corr, corr);
      l *= corr;
#pragma unroll
      for (int j = 0; j < NP; ++j) acc[j] = mul2(acc[j], c2);
      m = mx;
    }
    const float p0 = exp2f(s0 - m), p1 = exp2f(s1 - m);
    l += p0 + p1;
    vacc(vc0, p0 * sv0);
    vacc(vc1, p1 * sv1);
  };
#if KVQ_ATTN_PAIR_STAGES > 0
  int s_use = 0;
  for (uint32_t ob = uint32_t(32 * warp); ob < n_tok; ob += 256u) {
    issue(ob + 256u * (S - 1), s_use == 0 ? S - 1 : s_use - 1);
    cp_async_wait<S - 1>();  // this lane's copies of this iteration have landed
    const uint32_t st = stages + uint32_t(s_use * STAGE);
    s_use = s_use == S - 1 ? 0 : s_use + 1;
    if (ob + pp < n_tok) {  // a pair with no token left skips the work
      const bool two = ob + 16u + pp < n_tok;
      const uint4 kc0 = lds128(st + uint32_t(16 * lane));
      const uint4 kc1 = lds128(st + uint32_t(16 * (32 + lane)));
      const uint4 sc = lds128(st + uint32_t(2 * CB + 16 * lane));
      const uint4 vc0 = lds128(st + uint32_t(CB + 16 * lane));
      const uint4 vc1 = lds128(st + uint32_t(CB + 16 * (32 + lane)));
      const float part0 = kdot(kc0, __uint_as_float(sc.x));
      const float part1 = kdot(kc1, __uint_as_float(sc.z));
      const float s0 = part0 + __shfl_xor_sync(pmask, part0, 1);
      const float s1r = part1 + __shfl_xor_sync(pmask, part1, 1);
      update(s0, two ? s1r : -INFINITY, vc0, __uint_as_float(sc.y), vc1, __uint_as_float(sc.w));
    }
  }
  cp_async_wait<0>();
#else
  // two tokens per pair and iteration, t and t + kPairs: their eight loads
  // are issued together (a token past the block's range reads row t again
  // and gets weight 0)
  for (uint32_t o = uint32_t(threadIdx.x >> 1); o < n_tok; o += 2 * kPairs) {
    const uint32_t t0 = uint32_t(t_begin) + o;
    const bool two = o + kPairs < n_tok;
    const uint32_t t1 = two ? t0 + kPairs : t0;
    const uint4 kc0 = __ldg(reinterpret_cast<const uint4*>(kb + size_t(t0) * (D / 2)));
    const uint4 kc1 = __ldg(reinterpret_cast<const uint4*>(kb + size_t(t1) * (D / 2)));
    const float sk0 = __ldg(ks + size_t(t0) * ng), sk1 = __ldg(ks + size_t(t1) * ng);
    const uint4 vc0 = __ldg(reinterpret_cast<const uint4*>(vb + size_t(t0) * (D / 2)));
    const uint4 vc1 = __ldg(reinterpret_cast<const uint4*>(vb + size_t(t1) * (D / 2)));
    const float sv0 = __ldg(vs + size_t(t0) * ng), sv1 = __ldg(vs + size_t(t1) * ng);
    const float part0 = kdot(kc0, sk0), part1 = kdot(kc1, sk1);
    const float s0 = part0 + __shfl_xor_sync(pmask, part0, 1);
    const float s1r = part1 + __shfl_xor_sync(pmask, part1, 1);
    update(s0, two ? s1r : -INFINITY, vc0, sv0, vc1, sv1);
  }
#endif
  pdl_release();

  // ---- the warp's 16 pairs into one partial ----
  float mm = m;
#pragma unroll
  for (int o = 2; o <= 16; o <<= 1) mm = fmaxf(mm, __shfl_xor_sync(kFull, mm, o));
  const float f = m == -INFINITY ? 0.0f : exp2f(m - mm);
  float ls = l * f;
#pragma unroll
  for (int o = 2; o <= 16; o <<= 1) ls += __shfl_xor_sync(kFull, ls, o);
  float v[HC];
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    v[2 * j] = lo2(acc[j]) * f;
    v[2 * j + 1] = hi2(acc[j]) * f;
  }
  // reduce-scatter over lane bits 4..1 (the pair index): 32 -> 2 values,
  // lane keeps coordinates HC h + (lane & 30) + {0, 1}
#pragma unroll
  for (int o = 16, n = HC / 2; o >= 2; o >>= 1, n >>= 1) {
    const bool upper = lane & o;
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const float send = upper ? v[j] : v[j + n];
      const float keep = upper ? v[j + n] : v[j];
      v[j] = keep + __shfl_xor_sync(kFull, send, o);
    }
  }
  float* mine = s_part + warp * AP::FLOATS;
  mine[2 * NQ + HC * h + (lane & 30)] = v[0];
  mine[2 * NQ + HC * h + (lane & 30) + 1] = v[1];
  if (lane == 0) {
    mine[0] = mm;
    mine[1] = ls;
  }
  WideLane<D, ROT> L;
  L.init(a.signs, lane);
  attn_merge_store<D, ROT, NQ>(a, s_part, cluster, rank, nblk, head, warp, lane, L);
}

// ----------------------------- tensor-core decode attention (g = d, up to 8 queries) ---
//
// One scale per token (g = d), up to 4 queries per block and up to 8 per KV
// head (e.g. the Gemma-3-1B shape, d = 256 with 4 queries).  Per warp and chunk of 16
// tokens the rotated-domain scores and the accumulation run on the tensor
// cores (mma.sync):
//   scores           S = K Q^T:  m16n8k32, u8 x s8 -> s32.  M = 16 tokens,
//                                K = d rotated coordinates (d / 32 steps),
//                                N = 16 = 4 queries x 4 slices in two
//                                products of 8 columns;
//   accumulation     O^T = V^T P'^T:  m16n8k16, bf16 in, fp32 accumulate.
//                                M = d coordinates (d / 16 tiles), N = 8 = 4
//                                queries x (hi, lo), K = the 16 tokens.
// Scores: a code n enters as the byte q + 8 = n ^ 8 (one logic op per four
// codes) and the accumulator starts at -8 sum_i B[i], so the integer result
// is the exact product of the signed codes with the query slice B.  Each
// pre-scaled query is split into fixed point: exponent k with max |q| < 2^k
// and four signed 7-bit slices, q ~ 2^(k-6) (B_0 + B_1 2^-7 + B_2 2^-14 +
// B_3 2^-21), error at most 2^(k-28) <= 2^-27 max |q| per coordinate; the
// four exact integer products combine into the fp32 score.  Accumulation:
// int4 codes are exact in bf16; each weight p s_V is split into a bf16 high
// part and a bf16 remainder, the two columns of its pair, so products are
// exact and the two column sums carry ~16 significant bits (error ~2^-17
// relative, well under the fp16 output's).  With one scale per token (g = d)
// a token's K scale multiplies its score after the dot product and its V
// scale folds into its weight.
//
// Fragments (PTX ISA; lane = 4 g + c).  m16n8k32 with 8-bit inputs: A holds
// rows g and g + 8, columns 4c .. 4c + 3 and 16 + 4c .. 16 + 4c + 3 (four
// bytes a register); B rows (the K index) 4c .. 4c + 3 and 16 + 4c .. of
// column g.  m16n8k16 with 16-bit inputs: A rows g and g + 8, columns 2c,
// 2c + 1 and 2c + 8, 2c + 9; B rows 2c, 2c + 1, 2c + 8, 2c + 9 of column g.
// Both: C rows g, g + 8, columns 2c, 2c + 1.  The coordinates of a step may
// be any permutation applied to both operands: score step s of thread c
// takes the 32-bit word at byte c d/8 + 4s of tokens g and g + 8, its low
// nibbles (even coordinates) as K index 4c + i and its high nibbles (odd
// coordinates) as 16 + 4c + i; a V tile mt takes row g from the low nibble
// and row g + 8 from the high nibble of byte (d/16) g + mt.  Score column
// n = 2q + j: query q, slice j (2 + j in the second product); accumulation
// column n = 2q + h: query q, part h (0 high, 1 remainder).  So thread
// (g, c) holds the score of query c for tokens g and g + 8 and accumulates
// query c.

__device__ __forceinline__ void mma_bf16_m16n8k16(float (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// (lo, hi) -> bf16x2 with lo in the low half, rounded to nearest.
__device__ __forceinline__ uint32_t bf16x2_pack(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Constants of the nibble conversion kept in registers: with both operands
// of (x & mask) ^ c immediate the compiler emits two logic ops, with c in a
// register one three-input op.
struct TcConsts {
  uint32_t base, one, off, x8;
  __device__ __forceinline__ TcConsts()
      : base(0x43084308u), one(0x3F803F80u), off(0xC308C308u), x8(0x08080808u) {
    asm volatile("" : "+r"(base), "+r"(one), "+r"(off), "+r"(x8));  // opaque: stay in registers
  }
};

// The offset codes q + 8 = n ^ 8 of the low nibbles of the four bytes of x,
// one per byte: (x & 0x0F0F0F0F) ^ 0x08080808.
__device__ __forceinline__ uint32_t attn_tc_u8(uint32_t x, const TcConsts& k) {
  uint32_t t;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t) : "r"(x), "n"(0x0F0F0F0F), "r"(k.x8));
  return t;
}

// d = a b + c (first step of a chain) and d += a b, u8 x s8 -> s32
__device__ __forceinline__ void mma_u8s8_m16n8k32(int (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1, int c0, int c1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%10, %11, %10, %11};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c0), "r"(c1));
}
__device__ __forceinline__ void mma_u8s8_m16n8k32(int (&d)[4], uint32_t a0, uint32_t a1,
                                                  uint32_t a2, uint32_t a3, uint32_t b0,
                                                  uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2^n as fp32 for -126 <= n <= 127
__device__ __forceinline__ float attn_pow2(int n) { return __int_as_float((n + 127) << 23); }

// The codes of the low nibbles of bytes 0 and 2 of x as an exact bf16 pair:
// (x & 0x000F000F) ^ 0x43084308 is 128 + (n ^ 8) = 136 + q, minus 136.
__device__ __forceinline__ uint32_t attn_tc_lo(uint32_t x, const TcConsts& k) {
  uint32_t t;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(t) : "r"(x), "n"(0x000F000F), "r"(k.base));
  return bf16x2_fma(t, k.one, k.off);
}
// ... of the high nibbles of bytes 0 and 2 (shifted down first: bf16 has
// only 7 mantissa bits, so a nibble at bits 4-7 would reach the exponent).
__device__ __forceinline__ uint32_t attn_tc_hi(uint32_t x, const TcConsts& k) {
  return attn_tc_lo(x >> 4, k);
}

constexpr int kTcChunk = 16;   // tokens per warp and chunk
constexpr int kTcStages = 3;   // chunks in flight per warp
// staged chunk: K rows | V rows (16 x d/2 bytes; at d = 256 the 16-byte
// pieces are swizzled by the token index) | K scales | V scales
template <int D>
constexpr int tc_stage_bytes() {
  return 2 * kTcChunk * (D / 2) + 2 * kTcChunk * 4;
}
// position of 16-byte piece `ch` of staged row t
template <int D>
__device__ __forceinline__ int tc_piece(int t, int ch) {
  return D == 256 ? (ch ^ (t & 7)) : ch;
}
// `N` consecutive 32-bit words of a staged row from byte `b` (4N bytes
// within one 16-byte piece, or whole pieces)
template <int D, int N>
__device__ __forceinline__ void tc_lds_words(uint32_t row, int t, int b, uint32_t (&w)[N]) {
  if constexpr (N >= 4) {
#pragma unroll
    for (int k = 0; k < N / 4; ++k) {
      const uint4 v = lds128(row + uint32_t((tc_piece<D>(t, b / 16 + k) << 4)));
      w[4 * k] = v.x;
      w[4 * k + 1] = v.y;
      w[4 * k + 2] = v.z;
      w[4 * k + 3] = v.w;
    }
  } else if constexpr (N == 2) {
    const uint2 v = lds64(row + uint32_t((tc_piece<D>(t, b / 16) << 4) + (b % 16)));
    w[0] = v.x;
    w[1] = v.y;
  } else {
    w[0] = lds32(row + uint32_t((tc_piece<D>(t, b / 16) << 4) + (b % 16)));
  }
}

// QG: more than 4 queries per KV head, one grid row per (head, group of 4
// queries); else one grid row per head.  (Two resident blocks per SM up to
// d = 128: at most 128 registers.)
template <int D, int ROT, bool QG>
__global__ void __launch_bounds__(kAttnThreads, D <= 128 ? 2 : 1)
    kvq_attn_tc_kernel(const AttnArgs a) {
  namespace cg = cooperative_groups;
  constexpr int NQ = 4;
  constexpr int kTcRow = D / 2;               // code bytes per row
  constexpr int kTcStage = tc_stage_bytes<D>();
  constexpr int NS = D / 16;                  // accumulation tiles
  constexpr int KW = D / 32;                  // score steps = K words per thread and token
  constexpr int VW = D / 64;                  // V words per thread and token
  using P = Wide<D, ROT>;
  constexpr int W = P::W;
  using AP = AttnPartial<D, NQ>;
  extern __shared__ __align__(16) float s_part[];  // staging, queries; then merge slots

  pdl_wait();  // no global access before the previous kernel completes
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int nblk = int(cluster.num_blocks());
  // grid row = KV head, or (KV head, group of 4 queries): queries q0 .. q0 + qn - 1
  const int64_t head = QG ? blockIdx.y / a.qgroups : blockIdx.y;
  const int q0 = QG ? int(blockIdx.y - head * a.qgroups) * NQ : 0;
  const int qn = QG ? (a.nq - q0 < NQ ? a.nq - q0 : NQ) : a.nq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  // this block's tokens, then this warp's contiguous share (whole chunks)
  const int64_t per = (a.len + nblk - 1) / nblk;
  const int64_t t_begin = int64_t(rank) * per;
  const int64_t t_end = t_begin + per < a.len ? t_begin + per : a.len;
  const int64_t per_w =
      ((t_end - t_begin + kAttnWarps - 1) / kAttnWarps + kTcChunk - 1) / kTcChunk * kTcChunk;
  const int64_t w_begin = t_begin + int64_t(warp) * per_w;
  const int64_t w_end = w_begin + per_w < t_end ? w_begin + per_w : t_end;
  const int n_w = int(w_end > w_begin ? w_end - w_begin : 0);
  const int nchunk = (n_w + kTcChunk - 1) / kTcChunk;
  const uint8_t* kbase = a.k_packed + head * a.cap * kTcRow;
  const uint8_t* vbase = a.v_packed + head * a.cap * kTcRow;
  const float* ksc = a.k_scales + head * a.cap;
  const float* vsc = a.v_scales + head * a.cap;

  const uint32_t ring = smem_u32(s_part) + uint32_t(warp * kTcStages * kTcStage);
  // copy roles: a chunk's rows are copied in passes of RI rows, lane ->
  // (row lt + k RI, 16-byte piece lch) in pass k; whole chunks take fixed
  // per-lane offsets from running source pointers, the last partial chunk
  // the checked path
  constexpr int PR = kTcRow / 16;  // pieces per row
  constexpr int RI = 32 / PR;      // rows per pass
  constexpr int NPASS = kTcChunk / RI;
  const int lt = lane / PR, lch = lane % PR;
  uint32_t dsto[NPASS];
#pragma unroll
  for (int k = 0; k < NPASS; ++k) {
    const int t = lt + k * RI;
    dsto[k] = uint32_t(t * kTcRow + (tc_piece<D>(t, lch) << 4));
  }
  const uint8_t* kcur = kbase + (w_begin + lt) * kTcRow + lch * 16;
  const uint8_t* vcur = vbase + (w_begin + lt) * kTcRow + lch * 16;
  const float* scur = (lane < 16 ? ksc : vsc) + w_begin + (lane & 15);
  auto issue = [&](int ci) {  // called for ci = 0, 1, 2, ... in order
    if (ci < nchunk) {
      const uint32_t st = ring + uint32_t((ci % kTcStages) * kTcStage);
      const int rows = n_w - ci * kTcChunk < kTcChunk ? n_w - ci * kTcChunk : kTcChunk;
      if (rows == kTcChunk) {
#pragma unroll
        for (int k = 0; k < NPASS; ++k) {
          cp_async16(st + dsto[k], kcur + k * RI * kTcRow, 16);
          cp_async16(st + uint32_t(kTcChunk * kTcRow) + dsto[k], vcur + k * RI * kTcRow, 16);
        }
        cp_async4(st + uint32_t(2 * kTcChunk * kTcRow + lane * 4), scur, 4);
      } else {
        const int64_t r0 = w_begin + int64_t(ci) * kTcChunk;
#pragma unroll
        for (int i = lane; i < kTcChunk * PR; i += 32) {  // d / 64 pieces per lane
          const int t = i / PR, ch = i % PR;
          const bool ok = t < rows;
          const int64_t off = ok ? (r0 + t) * kTcRow + ch * 16 : r0 * kTcRow;
          const uint32_t dst = uint32_t(t * kTcRow + (tc_piece<D>(t, ch) << 4));
          cp_async16(st + dst, kbase + off, ok ? 16 : 0);
          cp_async16(st + uint32_t(kTcChunk * kTcRow) + dst, vbase + off, ok ? 16 : 0);
        }
        const int t = lane & 15;
        const bool ok = t < rows;
        const float* src = (lane < 16 ? ksc : vsc) + (ok ? r0 + t : r0);
        cp_async4(st + uint32_t(2 * kTcChunk * kTcRow + lane * 4), src, ok ? 4 : 0);
      }
      kcur += kTcChunk * kTcRow;
      vcur += kTcChunk * kTcRow;
      scur += kTcChunk;
    }
    cp_async_commit();  // possibly empty: keeps the group count uniform
  };
#pragma unroll
  for (int ci = 0; ci < kTcStages - 1; ++ci) issue(ci);

  // rotated, pre-scaled queries (score = <qr, y_K> in log2 units) in fixed
  // point: warp w rotates query w and splits it into its exponent k and four
  // 7-bit slices, stored after the staging rings as bytes [j][x & 1][x / 2]
  // (slice j, coordinate x), with k and the slice sums C_j beside them
  uint8_t* s_qs = reinterpret_cast<uint8_t*>(s_part + kAttnWarps * kTcStages * (kTcStage / 4));
  int* s_qk = reinterpret_cast<int*>(s_qs + NQ * 4 * D);  // [query][k, C_0 .. C_3, pad]
  float* s_p = reinterpret_cast<float*>(s_qk + NQ * 8);    // per warp: weights [4 queries][16 tokens]
  if (warp < NQ) {
    WideLane<D, ROT> L;  // (set up again for the merge: not live through the loop)
    L.init(a.signs, lane);
    uint32_t xw[P::C];
    if (warp < qn) {
      wide_load_words<D, ROT>(a.q + (head * a.nq + q0 + warp) * D, L, xw);
    } else {
#pragma unroll
      for (int j = 0; j < P::C; ++j) xw[j] = 0u;
    }
    float Y[W];
    wide_rotate_fwd<D, ROT>(xw, L, Y);
    float amax = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      Y[w] *= a.qscale;
      amax = fmaxf(amax, fabsf(Y[w]));
    }
#pragma unroll
    for (int msk = 1; msk <= 16; msk <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, msk));
    // max |q| < 2^k (k clamped so that every power of two below is normal)
    const int k = min(max(int((__float_as_uint(amax) >> 23) & 0xFFu) - 126, -90), 120);
    const float up = attn_pow2(6 - k);
    uint8_t* qs = s_qs + warp * 4 * D;
    int csum[4] = {0, 0, 0, 0};
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const int x = L.k2 * W + w;
      float t = Y[w] * up;  // |t| < 64; each step below is exact
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float b = rintf(t);
        csum[j] += int(b);
        qs[(2 * j + (x & 1)) * (D / 2) + (x >> 1)] = uint8_t(int(b) & 0xFF);
        t = (t - b) * 128.0f;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int msk = 1; msk <= 16; msk <<= 1) csum[j] += __shfl_xor_sync(kFull, csum[j], msk);
    if (lane == 0) {
      s_qk[warp * 8] = k;
#pragma unroll
      for (int j = 0; j < 4; ++j) s_qk[warp * 8 + 1 + j] = csum[j];
    }
  }
  __syncthreads();
  // B operands of the scores: column g = 2 q + j of query q = g / 2, slice j
  // (qa) and 2 + j (qc); step s holds the slices of even coordinates 2m and
  // odd 2m + 1, m = c d/8 + 4s .. + 3
  uint32_t qa[KW][2], qc[KW][2];
  {
    const uint8_t* qs = s_qs + (g >> 1) * 4 * D;
    const int j = g & 1;
#pragma unroll
    for (int s = 0; s < KW; ++s) {
      const int m0 = (D / 8) * c + 4 * s;
#pragma unroll
      for (int par = 0; par < 2; ++par) {
        qa[s][par] = *reinterpret_cast<const uint32_t*>(qs + (2 * j + par) * (D / 2) + m0);
        qc[s][par] = *reinterpret_cast<const uint32_t*>(qs + (2 * (j + 2) + par) * (D / 2) + m0);
      }
    }
  }
  // query c's exponent and the accumulators' start values -8 C_j
  const float f_hi = attn_pow2(s_qk[c * 8] - 13), f_lo = attn_pow2(s_qk[c * 8] - 27);
  const int ca0 = -8 * s_qk[c * 8 + 1], ca1 = -8 * s_qk[c * 8 + 2];
  const int cc0 = -8 * s_qk[c * 8 + 3], cc1 = -8 * s_qk[c * 8 + 4];

  float m = -INFINITY, l = 0.0f;  // of query c
  float o[NS][4];  // O^T tiles: coordinates 2 ((d/16) g + mt) (+1), columns 2c, 2c + 1
#pragma unroll
  for (int mt = 0; mt < NS; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[mt][i] = 0.0f;
  const uint32_t pw = smem_u32(s_p) + uint32_t(warp * NQ * kTcChunk * 4);
  const TcConsts kc;

  for (int ci = 0; ci < nchunk; ++ci) {
    cp_async_wait<kTcStages - 2>();
    __syncwarp();  // the chunk's copies (by every lane) are visible
    const uint32_t st = ring + uint32_t((ci % kTcStages) * kTcStage);
    const uint32_t kst = st, vst = st + uint32_t(kTcChunk * kTcRow);
    const uint32_t sst = st + uint32_t(2 * kTcChunk * kTcRow);
    const int rows = n_w - ci * kTcChunk < kTcChunk ? n_w - ci * kTcChunk : kTcChunk;

    // ---- scores: tokens g and g + 8, query c ----
    int sa[4], sc[4];  // slices (0, 1) and (2, 3): exact integer products
    {  // bytes [c d/8, (c + 1) d/8) of tokens g and g + 8
      uint32_t w0[KW], w8[KW];
      tc_lds_words<D, KW>(kst + uint32_t(g * kTcRow), g, (D / 8) * c, w0);
      tc_lds_words<D, KW>(kst + uint32_t((g + 8) * kTcRow), g + 8, (D / 8) * c, w8);
#pragma unroll
      for (int s = 0; s < KW; ++s) {
        const uint32_t a0 = attn_tc_u8(w0[s], kc), a1 = attn_tc_u8(w8[s], kc);
        const uint32_t a2 = attn_tc_u8(w0[s] >> 4, kc), a3 = attn_tc_u8(w8[s] >> 4, kc);
        if (s == 0) {
          mma_u8s8_m16n8k32(sa, a0, a1, a2, a3, qa[0][0], qa[0][1], ca0, ca1);
          mma_u8s8_m16n8k32(sc, a0, a1, a2, a3, qc[0][0], qc[0][1], cc0, cc1);
        } else {
          mma_u8s8_m16n8k32(sa, a0, a1, a2, a3, qa[s][0], qa[s][1]);
          mma_u8s8_m16n8k32(sc, a0, a1, a2, a3, qc[s][0], qc[s][1]);
        }
      }
    }
    const float sk0 = __uint_as_float(lds32(sst + uint32_t(g * 4)));
    const float sk8 = __uint_as_float(lds32(sst + uint32_t((g + 8) * 4)));
    // 2^(k-6) (B_0 + B_1 2^-7 + ...): the slice pairs combine exactly in
    // integers (|sum| < 2^25), then in fp32
    const float sc0 =
        g < rows ? fmaf(float(sc[0] * 128 + sc[1]), f_lo, float(sa[0] * 128 + sa[1]) * f_hi) * sk0
                 : -INFINITY;
    const float sc8 =
        g + 8 < rows ? fmaf(float(sc[2] * 128 + sc[3]), f_lo, float(sa[2] * 128 + sa[3]) * f_hi) * sk8
                     : -INFINITY;

    // ---- online softmax of query c over the chunk (lanes c, c + 4, ...) ----
    // lazy maximum (kAttnSlack)
    float mx = fmaxf(sc0, sc8);
#pragma unroll
    for (int msk = 4; msk <= 16; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, msk));
    if (__any_sync(kFull, mx > m + kAttnSlack)) {  // always on the first chunk (m = -inf)
      const float m_new = mx > m + kAttnSlack ? mx : m;  // finite: the chunk holds a valid token
      const float corr = exp2f(m - m_new);
      l *= corr;
#pragma unroll
      for (int mt = 0; mt < NS; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[mt][i] *= corr;
      m = m_new;
    }
    const float p0 = exp2f(sc0 - m), p8 = exp2f(sc8 - m);
    float ps = p0 + p8;
#pragma unroll
    for (int msk = 4; msk <= 16; msk <<= 1) ps += __shfl_xor_sync(kFull, ps, msk);
    l += ps;
    // weights p s_V by (query, token) through shared memory, then the B
    // operand: column g = 2 q + h, tokens 2c, 2c + 1 and 2c + 8, 2c + 9
    const float sv0 = __uint_as_float(lds32(sst + uint32_t((kTcChunk + g) * 4)));
    const float sv8 = __uint_as_float(lds32(sst + uint32_t((kTcChunk + g + 8) * 4)));
    sts32(pw + uint32_t((c * kTcChunk + g) * 4), __float_as_uint(p0 * sv0));
    sts32(pw + uint32_t((c * kTcChunk + g + 8) * 4), __float_as_uint(p8 * sv8));
    __syncwarp();
    uint32_t pb[2];
    {
      const bool rem = g & 1;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const uint2 v = lds64(pw + uint32_t(((g >> 1) * kTcChunk + 2 * c + 8 * r) * 4));
        const float v0 = __uint_as_float(v.x), v1 = __uint_as_float(v.y);
        const uint32_t hi = bf16x2_pack(v0, v1);
        const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xFFFF0000u);
        pb[r] = rem ? bf16x2_pack(v0 - h0, v1 - h1) : hi;
      }
    }

    // ---- accumulation: V rows 2c, 2c + 1, 2c + 8, 2c + 9, bytes [(d/16) g, +d/16) ----
    {
      uint32_t wa[VW], wb[VW], wc[VW], wd[VW];
      tc_lds_words<D, VW>(vst + uint32_t(2 * c * kTcRow), 2 * c, (D / 16) * g, wa);
      tc_lds_words<D, VW>(vst + uint32_t((2 * c + 1) * kTcRow), 2 * c + 1, (D / 16) * g, wb);
      tc_lds_words<D, VW>(vst + uint32_t((2 * c + 8) * kTcRow), 2 * c + 8, (D / 16) * g, wc);
      tc_lds_words<D, VW>(vst + uint32_t((2 * c + 9) * kTcRow), 2 * c + 9, (D / 16) * g, wd);
#pragma unroll
      for (int mt = 0; mt < NS; ++mt) {
        const uint32_t sel = uint32_t(mt & 3) | (uint32_t(4 + (mt & 3)) << 8);
        const uint32_t x01 = __byte_perm(wa[mt >> 2], wb[mt >> 2], sel);  // tokens 2c, 2c + 1
        const uint32_t x89 = __byte_perm(wc[mt >> 2], wd[mt >> 2], sel);  // 2c + 8, 2c + 9
        mma_bf16_m16n8k16(o[mt], attn_tc_lo(x01, kc), attn_tc_hi(x01, kc), attn_tc_lo(x89, kc),
                          attn_tc_hi(x89, kc), pb[0], pb[1]);
      }
    }
    __syncwarp();  // the stage and the weights are consumed before they are refilled
    issue(ci + kTcStages - 1);
  }
  cp_async_wait<0>();
  pdl_release();
  __syncthreads();  // the staging rings become the merge area

  // ---- this warp's partial into its merge slot (y order) ----
  float* mine = s_part + warp * AP::FLOATS;
  if (g == 0) {
    mine[2 * c] = m;
    mine[2 * c + 1] = l;
  }
#pragma unroll
  for (int mt = 0; mt < NS; ++mt) {
    const int y = 2 * ((D / 16) * g + mt);
    mine[2 * NQ + c * D + y] = o[mt][0] + o[mt][1];
    mine[2 * NQ + c * D + y + 1] = o[mt][2] + o[mt][3];
  }
  WideLane<D, ROT> L;
  L.init(a.signs, lane);
  if constexpr (QG) {
    attn_merge_store<D, ROT, NQ>(a, s_part, cluster, rank, nblk, head, warp, lane, L, q0, qn);
  } else {
    attn_merge_store<D, ROT, NQ>(a, s_part, cluster, rank, nblk, head, warp, lane, L);
  }
}

// Dynamic shared memory of kvq_attn_tc_kernel.
template <int D>
constexpr int attn_tc_smem_bytes() {
  constexpr int merge = (kAttnWarps * AttnPartial<D, 4>::FLOATS + 2 * 4) * 4;
  constexpr int staging = kAttnWarps * kTcStages * tc_stage_bytes<D>() + 4 * 4 * D + 4 * 8 * 4 +
                          kAttnWarps * 4 * kTcChunk * 4;
  return merge > staging ? merge : staging;
}

// Dynamic shared memory of kvq_attn_kernel.
template <int D, int NQ>
constexpr int attn_smem_bytes() {
  constexpr int merge = (kAttnWarps * AttnPartial<D, NQ>::FLOATS + 2 * NQ) * 4;
  constexpr int staging = kAttnWarps * kAttnStages * attn_chunk_bytes<D>() + NQ * D * 4;
  return merge > staging ? merge : staging;
}

}  // namespace kvq
