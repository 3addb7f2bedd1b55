// Sparse attention for decoding shapes: a few query rows per sequence, so a
// tile holds the GQA group's q heads x rows = at most 16 query vectors of one
// kv head.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — the pooled
// K/V of the selected documents joined to the K/V of the query's recent context;
// Parallel (document-wise) RoPE and Global RoPE offset by k (Figure 2)]
//
// Same result as the other attention kernels. A decoding step attends over a
// few hundred keys per head (a few MB per layer at 4 flop per byte), so its
// time is the chain of dependent memory round trips plus the latency of the
// instructions each warp issues; neither bandwidth nor arithmetic throughput
// bounds it. The kernel keeps that chain short:
//  - A CTA (one per SM) owns one kv head, one tile of query vectors and one
//    split of the key list: an even share of the sequence's memory keys (the
//    selected pooled rows) and of its local keys (the recent context, rotated
//    by rope_rows and stored there as bf16 high and low halves).
//  - Inside the CTA every warp is an independent flash-decoding worker: the
//    share is cut into steps of 16 keys and warp w takes steps w, w + 8, ...
//    Each warp copies its own steps' rows by cp.async into its own two
//    shared-memory stages (the next step in flight while one is computed; a
//    key's bank row is read from the selection list a step before its copy),
//    keeps its own running max, sum and output, and synchronises with no
//    other warp until the end.
//  - A step is two warp-level bf16 MMA chains (m16n8k16, fp32 accumulate), the
//    16-vector tile as M: S = Q K^T (queries split into bf16 high + low parts,
//    local keys too, so the logits keep fp32 accuracy), then O += P V with P
//    taken straight from S's accumulators as the A operand (rounded to bf16).
//  - At the end the 8 warps' (o, m, l) are merged through shared memory; with
//    several splits per (tile, kv head) each CTA then writes an unnormalised
//    partial and the last to finish (atomic ticket, no waiting) merges them.
#include <math.h>

#include "attend_params.cuh"

namespace msa {
namespace {

constexpr int kDThreads = 256;                     // 8 warps
constexpr int kDWarps = kDThreads / 32;
constexpr int kStepKeys = 16;                      // keys per warp step (the K of P.V)
constexpr int kRowB = 272;                         // bytes per staged bf16 row (256 + 16)
constexpr int kTileV = 16;                         // query vectors per tile (MMA M)
constexpr int offSK = 0;                           // within a stage: keys (bf16, or the high halves)
constexpr int offSL = offSK + kStepKeys * kRowB;   // low halves of local keys
constexpr int offSV = offSL + kStepKeys * kRowB;   // values
constexpr int kStageB = offSV + kStepKeys * kRowB; // 13,056 B
constexpr int kWarpB = 2 * kStageB;                // two stages per warp
constexpr int offQhi = kDWarps * kWarpB;           // queries [16][272 B], high and low parts
constexpr int offQlo = offQhi + kTileV * kRowB;
constexpr int kDecSmem = offQlo + kTileV * kRowB;  // 217,600 B
// end-of-CTA merge, over the warps' stages: o [8 warps][16][132] fp32 (rows padded: the
// fragment stores of a warp hit distinct banks), then m, l [8][16]
constexpr int kMRow = kHeadDim + 4;
constexpr int offMO = 0;
constexpr int offMM = offMO + kDWarps * kTileV * kMRow * 4;
constexpr int offMLs = offMM + kDWarps * kTileV * 4;
static_assert(offMLs + kDWarps * kTileV * 4 <= offQhi, "the merge fits the stages");
static_assert(kDecSmem <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ uint32_t saddr(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D += A B for one m16n8k16 tile (A row-major 16x16, B column-major 16x8), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf_round_f(float x) { return __uint_as_float(f2bf_bits(x) << 16); }

__global__ void __launch_bounds__(kDThreads, 1) attend_dec_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = lane >> 2, c = lane & 3;  // MMA fragment coordinates
  const int sp = blockIdx.x, kvh = blockIdx.y, tile = blockIdx.z;
  const int s = seq_of(p.tile_off, p.n_seq, tile);
  const int row0 = p.q_seq_off[s] + (tile - p.tile_off[s]) * p.rt;
  const int nr = min(p.rt, p.q_seq_off[s + 1] - row0);
  const int nvec = nr * p.group;                           // valid query vectors (<= 16)
  const int g0 = p.q_start[s] + (row0 - p.q_seq_off[s]);  // active index of the tile's first row
  const int n_loc_s = p.loc_off[s + 1] - p.loc_off[s];
  const int lvis = max(0, min(n_loc_s, g0 + nr));          // local keys visible to the tile's last row
  const size_t row_stride = (size_t)p.hkv * kHeadDim;
  const float sl2 = p.scale * 1.4426950408889634f;         // logits in log2 units
  // active-context index of MMA rows g and g + 8 (-1: padding, sees nothing)
  const int ga = g < nvec ? g0 + g / p.group : -1;
  const int gb = g + 8 < nvec ? g0 + (g + 8) / p.group : -1;

  pdl_wait();  // the selection (gather) and the rotated rows (rope_rows) come from earlier kernels
  pdl_trigger();

  // ---- query tile (16 vectors v = rr * group + gg; past nvec zero): its loads go out
  // together with those of the key ranges below
  const int qv_v = tid >> 4, qv_d0 = 8 * (tid & 15);
  float4 qa = make_float4(0.f, 0.f, 0.f, 0.f), qb = qa;
  if (qv_v < nvec) {
    const int rr = qv_v / p.group, gg = qv_v - rr * p.group;
    const float4* qv = reinterpret_cast<const float4*>(
        p.qrot + ((size_t)(row0 + rr) * p.hq + kvh * p.group + gg) * kHeadDim + qv_d0);
    qa = __ldcg(qv);
    qb = __ldcg(qv + 1);
  }

  // ---- this split's share of the memory keys [m0, m1) and of the local keys [l0, l1)
  const int64_t mem_base = __ldcg(p.sel_off + s);
  const int64_t n_mem = __ldcg(p.sel_off + s + 1) - mem_base;
  const int64_t pm = (n_mem + p.n_splits - 1) / p.n_splits;
  const int64_t m0 = min(n_mem, (int64_t)sp * pm), m1 = min(n_mem, m0 + pm);
  const int pl = (lvis + p.n_splits - 1) / p.n_splits;
  const int l0 = min(lvis, sp * pl), l1 = min(lvis, l0 + pl);
  const int nsm = (int)((m1 - m0 + kStepKeys - 1) / kStepKeys);  // memory steps, then local steps
  const int nsteps = nsm + (l1 - l0 + kStepKeys - 1) / kStepKeys;

  // ---- this warp's steps w, w + 8, ...: lane kl < 16 looks up the bank row of key kl of a
  // step; copy instruction u then moves rows 2u and 2u + 1 whole (lanes 0-15 and 16-31, 16 B
  // each), so every instruction reads two contiguous 256-byte rows
  const int kl = lane & 15;
  uint8_t* wst = sm + w * kWarpB;
  auto row_of = [&](int i) -> int64_t {  // bank row (memory) or local row of key kl in step i; -1: none
    if (i >= nsteps) return -1;
    if (i < nsm) {
      const int64_t key = m0 + (int64_t)i * kStepKeys + kl;
      if (key >= m1) return -1;
      return p.sel_chunk ? __ldcg(p.sel_chunk + mem_base + key) : mem_base + key;
    }
    const int key = l0 + (i - nsm) * kStepKeys + kl;
    return key < l1 ? (int64_t)(p.loc_off[s] + key) : -1;
  };
  auto issue = [&](int i, int64_t r_mine, int stage) {
    if (i < nsteps) {
      uint8_t* stg = wst + stage * kStageB;
      const bool loc = i >= nsm;
      const int piece = 16 * (lane & 15);
#pragma unroll
      for (int u = 0; u < kStepKeys / 2; ++u) {
        const int key = 2 * u + (lane >> 4);
        const int64_t r = __shfl_sync(0xffffffffu, r_mine, key);
        const int so = key * kRowB + piece;
        if (r >= 0) {
          if (!loc) {
            const size_t off = ((size_t)r * row_stride + (size_t)kvh * kHeadDim) * 2 + piece;
            cp16(saddr(stg + offSK + so), reinterpret_cast<const uint8_t*>(p.mem_k) + off);
            cp16(saddr(stg + offSV + so), reinterpret_cast<const uint8_t*>(p.mem_v) + off);
          } else {
            const size_t lrow = (size_t)r * p.hkv + kvh;
            const uint8_t* kr = reinterpret_cast<const uint8_t*>(p.krot) + lrow * 512;  // high, then low halves
            cp16(saddr(stg + offSK + so), kr + piece);
            cp16(saddr(stg + offSL + so), kr + 256 + piece);
            cp16(saddr(stg + offSV + so), reinterpret_cast<const uint8_t*>(p.v_loc + lrow * kHeadDim) + piece);
          }
        } else {
          // a key past the range: zero values (P is 0 there, and 0 x NaN would not be)
          *reinterpret_cast<uint4*>(stg + offSV + so) = make_uint4(0, 0, 0, 0);
        }
      }
    }
    cp_commit();
  };
  int64_t r_next;  // bank row of key kl in the warp's third step
  {
    const int64_t r0 = row_of(w), r1 = row_of(w + kDWarps), r2 = row_of(w + 2 * kDWarps);
    issue(w, r0, 0);
    issue(w + kDWarps, r1, 1);
    r_next = r2;
  }

  // ---- queries as bf16 high and low parts (shared by the warps)
  {
    const float f[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    float h[8], l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      h[i] = bf_round_f(f[i]);
      l[i] = f[i] - h[i];
    }
    *reinterpret_cast<uint4*>(sm + offQhi + qv_v * kRowB + 2 * qv_d0) =
        make_uint4(pack_bf2(h[0], h[1]), pack_bf2(h[2], h[3]), pack_bf2(h[4], h[5]), pack_bf2(h[6], h[7]));
    *reinterpret_cast<uint4*>(sm + offQlo + qv_v * kRowB + 2 * qv_d0) =
        make_uint4(pack_bf2(l[0], l[1]), pack_bf2(l[2], l[3]), pack_bf2(l[4], l[5]), pack_bf2(l[6], l[7]));
  }
  __syncthreads();

  // Q as the A operand of S, all 8 k-steps (16 dims each), high and low parts: held in
  // registers for every step of the warp
  uint32_t qh[8][4], ql[8][4];
  {
    const int arow = ((lane >> 3) & 1) * 8 + (lane & 7), acol = (lane >> 4) * 8;
    const uint32_t aQhi = saddr(sm + offQhi + arow * kRowB + 2 * acol);
    const uint32_t aQlo = saddr(sm + offQlo + arow * kRowB + 2 * acol);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      ldsm_x4(aQhi + 32 * ks, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3]);
      ldsm_x4(aQlo + 32 * ks, ql[ks][0], ql[ks][1], ql[ks][2], ql[ks][3]);
    }
  }
  // B of S for key n-tile nt: keys 8nt + (lane & 7), matrix i = dims 8i..8i+7 of a 32-dim chunk
  const int brow = lane & 7, bcol = (lane >> 3) * 8;
  // B of O (V^T via .trans) for dims 16j..16j+15: matrix i = keys + 8(i & 1), dims + 8(i >> 1)
  const int vrow = ((lane >> 3) & 1) * 8 + (lane & 7), vcol = (lane >> 4) * 8;

  float o[16][4];  // O: 16 vectors x 128 dims; n-tile n = dims 8n..8n+7
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;  // running max / sum of rows g, g + 8

  int it = 0;
  for (int i = w; i < nsteps; i += kDWarps, ++it) {
    const int stage = it & 1;
    cp_wait<1>();  // this step's copies (this lane's); the next step's may still be in flight
    __syncwarp();  // ... and every lane's
    const uint8_t* stg = wst + stage * kStageB;
    const bool loc = i >= nsm;
    const int64_t kb = loc ? l0 + (int64_t)(i - nsm) * kStepKeys : m0 + (int64_t)i * kStepKeys;
    const int nk = (int)min((int64_t)kStepKeys, (loc ? l1 : m1) - kb);

    // ---- S (16 vectors x 16 keys) = Q K^T: n-tiles 0 (keys 0-7) and 1 (keys 8-15), each
    // accumulated in two halves (even and odd k-steps) so that four MMA chains run side by side
    float sa[2][4], sb[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = 0.f;
#pragma unroll
    for (int k2 = 0; k2 < 4; ++k2) {  // 32 dims: k-steps 2k2 and 2k2 + 1
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(saddr(stg + offSK + (8 * nt + brow) * kRowB + 2 * (32 * k2 + bcol)), b0, b1, b2, b3);
        mma16816(sa[nt], qh[2 * k2], b0, b1);
        mma16816(sb[nt], qh[2 * k2 + 1], b2, b3);
        mma16816(sa[nt], ql[2 * k2], b0, b1);
        mma16816(sb[nt], ql[2 * k2 + 1], b2, b3);
        if (loc) {
          ldsm_x4(saddr(stg + offSL + (8 * nt + brow) * kRowB + 2 * (32 * k2 + bcol)), b0, b1, b2, b3);
          mma16816(sa[nt], qh[2 * k2], b0, b1);
          mma16816(sb[nt], qh[2 * k2 + 1], b2, b3);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[nt][e] += sb[nt][e];
    // ---- mask (log2 units), online softmax over this step's keys. sa[nt]: rows g (0, 1) and
    // g + 8 (2, 3), keys 8nt + 2c, + 1
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int jk = 8 * nt + 2 * c + (e & 1);
        const int gr = e < 2 ? ga : gb;
        const bool vis = jk < nk && gr >= 0 && (!loc || kb + jk <= gr);
        sa[nt][e] = vis ? sa[nt][e] * sl2 : -INFINITY;
      }
    float xA = fmaxf(fmaxf(sa[0][0], sa[0][1]), fmaxf(sa[1][0], sa[1][1]));
    float xB = fmaxf(fmaxf(sa[0][2], sa[0][3]), fmaxf(sa[1][2], sa[1][3]));
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
      xA = fmaxf(xA, __shfl_xor_sync(0xffffffffu, xA, x));
      xB = fmaxf(xB, __shfl_xor_sync(0xffffffffu, xB, x));
    }
    const float nA = fmaxf(mA, xA), nB = fmaxf(mB, xB);
    const float cA = nA == -INFINITY ? 1.f : exp2f(mA - nA);
    const float cB = nB == -INFINITY ? 1.f : exp2f(mB - nB);
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pr[nt][0] = nA == -INFINITY ? 0.f : exp2f(sa[nt][0] - nA);
      pr[nt][1] = nA == -INFINITY ? 0.f : exp2f(sa[nt][1] - nA);
      pr[nt][2] = nB == -INFINITY ? 0.f : exp2f(sa[nt][2] - nB);
      pr[nt][3] = nB == -INFINITY ? 0.f : exp2f(sa[nt][3] - nB);
    }
    float sA = pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1], sB = pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
      sA += __shfl_xor_sync(0xffffffffu, sA, x);
      sB += __shfl_xor_sync(0xffffffffu, sB, x);
    }
    lA = lA * cA + sA;
    lB = lB * cB + sB;
    mA = nA;
    mB = nB;
    // P as the A operand of P.V (16 vectors x 16 keys): the accumulator layout of S's two n-tiles
    const uint32_t pa[4] = {pack_bf2(pr[0][0], pr[0][1]), pack_bf2(pr[0][2], pr[0][3]), pack_bf2(pr[1][0], pr[1][1]),
                            pack_bf2(pr[1][2], pr[1][3])};

    // ---- O = O * corr + P V over the 128 dims (16 n-tiles of 8); most steps leave the max in place
    if (__any_sync(0xffffffffu, cA != 1.f || cB != 1.f)) {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= cA; o[n][1] *= cA;
        o[n][2] *= cB; o[n][3] *= cB;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(saddr(stg + offSV + vrow * kRowB + 2 * (16 * j + vcol)), v0, v1, v2, v3);
      mma16816(o[2 * j], pa, v0, v1);
      mma16816(o[2 * j + 1], pa, v2, v3);
    }
    __syncwarp();  // every lane is done with this stage
    // the warp's step after next goes into this stage
    issue(i + 2 * kDWarps, r_next, stage);
    r_next = row_of(i + 3 * kDWarps);
  }
  cp_wait<0>();
  __syncthreads();  // every warp is done with its stages: they hold the merge now

  // ---- merge the 8 warps: o [w][v][d], m and l [w][v]
  float* mo = reinterpret_cast<float*>(sm + offMO);
  float* mm = reinterpret_cast<float*>(sm + offMM);
  float* ml = reinterpret_cast<float*>(sm + offMLs);
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int d = 8 * n + 2 * c;
    *reinterpret_cast<float2*>(mo + (w * kTileV + g) * kMRow + d) = make_float2(o[n][0], o[n][1]);
    *reinterpret_cast<float2*>(mo + (w * kTileV + g + 8) * kMRow + d) = make_float2(o[n][2], o[n][3]);
  }
  if (c == 0) {
    mm[w * kTileV + g] = mA;
    mm[w * kTileV + g + 8] = mB;
    ml[w * kTileV + g] = lA;
    ml[w * kTileV + g + 8] = lB;
  }
  __syncthreads();
  const int d = tid & (kHeadDim - 1);
  const bool split = p.n_splits > 1;
  for (int v = tid >> 7; v < nvec; v += 2) {
    float m = -INFINITY;
#pragma unroll
    for (int x = 0; x < kDWarps; ++x) m = fmaxf(m, mm[x * kTileV + v]);
    float l = 0.f, r = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int x = 0; x < kDWarps; ++x) {
        const float wt = exp2f(mm[x * kTileV + v] - m);  // 0 for a warp that saw nothing
        l += ml[x * kTileV + v] * wt;
        r += mo[(x * kTileV + v) * kMRow + d] * wt;
      }
    }
    const int rr = v / p.group, gg = v - rr * p.group;
    const size_t rh = (size_t)(row0 + rr) * p.hq + kvh * p.group + gg;
    if (!split) {
      const float res = l > 0.f ? r / l : 0.f;
      p.out[rh * kHeadDim + d] = (uint16_t)f2bf_bits(res);
      if (p.out_f32) p.out_f32[rh * kHeadDim + d] = res;
      if (p.lse && d == 0) p.lse[rh] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else {
      const size_t pi = rh * p.n_splits + sp;
      p.part_o[pi * kHeadDim + d] = r;
      if (d == 0) p.part_ml[pi] = make_float2(m, l);
    }
  }
  if (!split) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(p.tickets + (size_t)tile * p.hkv + kvh, 1u) == (unsigned)(p.n_splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // ---- the last CTA of this (tile, kv head) merges every split (log2 units)
  for (int v = tid >> 7; v < nvec; v += 2) {
    const int rr = v / p.group, gg = v - rr * p.group;
    const size_t rh = (size_t)(row0 + rr) * p.hq + kvh * p.group + gg;
    float mx = -INFINITY;
    for (int j = 0; j < p.n_splits; ++j) {
      const float2 x = __ldcg(p.part_ml + rh * p.n_splits + j);
      if (x.y > 0.f) mx = fmaxf(mx, x.x);
    }
    float wsum = 0.f, r = 0.f;
    for (int j = 0; j < p.n_splits; ++j) {
      const float2 x = __ldcg(p.part_ml + rh * p.n_splits + j);
      if (!(x.y > 0.f)) continue;
      const float wt = exp2f(x.x - mx);
      wsum += x.y * wt;
      r += wt * __ldcg(p.part_o + (rh * p.n_splits + j) * kHeadDim + d);
    }
    r = wsum > 0.f ? r / wsum : 0.f;
    p.out[rh * kHeadDim + d] = (uint16_t)f2bf_bits(r);
    if (p.out_f32) p.out_f32[rh * kHeadDim + d] = r;
    if (p.lse && d == 0) p.lse[rh] = wsum > 0.f ? (mx + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
  }
}

}  // namespace

msa_status launch_attend_dec(const AttnParams& P, int vec, cudaStream_t st) {
  (void)vec;  // the tile is always 16 MMA rows; P.rt rows x P.group heads of them are used
  static std::atomic<uint64_t> attr{0};
  cudaError_t e = smem_limit_once(attend_dec_kernel, kDecSmem, attr);
  if (e != cudaSuccess) return cuda_fail(e, "attend: decoding kernel shared memory");
  e = launch_pdl(attend_dec_kernel, dim3((unsigned)P.n_splits, (unsigned)P.hkv, (unsigned)P.n_tiles),
                 dim3(kDThreads), (size_t)kDecSmem, st, P);
  if (e != cudaSuccess) return cuda_fail(e, "attend: decoding kernel");
  return launch_check("attend: decoding kernel");
}

}  // namespace msa
