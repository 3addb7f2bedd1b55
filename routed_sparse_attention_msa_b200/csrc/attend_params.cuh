// Parameter block shared by the attention kernels (split-K decoding in
// attend.cu, the tensor-core kernel for many query rows in attend_tc.cu), and
// the host-side hooks between them.
#pragma once

#include "msa_internal.cuh"

namespace msa {

struct AttnParams {
  const uint16_t* q;
  const uint16_t* k_loc;
  const uint16_t* v_loc;
  const uint16_t* mem_k;
  const uint16_t* mem_v;
  const int64_t* sel_off;        // nullptr: the routed form below
  const int64_t* sel_chunk;
  const int32_t* top_ids;        // routed form: [n_seq, top_k] selected documents
  const int64_t* doc_chunk_off;  // routed form: [n_docs + 1] each document's chunk range
  int64_t n_docs, max_sel;
  int top_k;
  int rot_in_kernel;  // decoding kernel: 1 = it rotates its local keys itself, 0 = rope_rows did
  int rope_q;         // 1: rope_rows rotates the query rows (0: the decoding kernel does)
  float* qrot;      // [n_q, hq, d]
  float* krot;      // [n_loc, hkv, d], or [n_loc, hkv] rows of 512 B with krot_split
  float* part_o;    // [n_q, hq, splits, d]
  float2* part_ml;  // [n_q, hq, splits]
  unsigned* tickets;  // [n_tiles * hkv]
  uint16_t* out;
  float* out_f32;
  float* lse;
  int n_seq, n_q, n_loc, hq, hkv, group, rt, n_splits, n_tiles;
  int krot_split;  // 1: rope_rows stores each rotated local key as bf16 high halves then low halves (512 B)
  float scale;
  double pos_offset, log2_theta;
  double inv_freq[kHeadDim / 2];  // RoPE frequency of pair i: theta^(-2i/d), formed on the host in double
  int32_t q_seq_off[kMaxSeq + 1];
  int32_t q_start[kMaxSeq];
  int32_t loc_off[kMaxSeq + 1];
  int32_t tile_off[kMaxSeq + 1];
};

// An angle (radians, double) reduced to [-pi, pi] in double, as a float: sincosf
// then evaluates it on its short, accurate range for positions of any size.
__device__ __forceinline__ float reduced_angle(double ang) {
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  return (float)(ang - two_pi * rint(ang * inv_two_pi));
}

// Index of the segment of `off` (n_seq + 1 ascending offsets) holding x.
__device__ __forceinline__ int seq_of(const int32_t* off, int n_seq, int x) {
  int lo = 0, hi = n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// attend_tc.cu: one CTA per (tile of 128 query vectors = rt rows x group q
// heads, kv head, key split); grid (n_tiles, hkv, n_splits), the splits of a
// (tile, kv head) one cluster. Needs rope_rows to have run with krot_split =
// 1; lists the routed form's memory rows itself when top_k <= kDecRoutedMaxK.
constexpr int kAttnTcVec = 128;
msa_status launch_attend_tc(const AttnParams& P, cudaStream_t st);
int attend_tc_error_take();  // 1 if its bounded wait ran out since the last call

// attend_dec_tc.cu: the decoding shapes (at most 16 query vectors per CTA) on
// the tensor cores, keys as the MMA's M side; same grid and split-K plan as
// the split-K kernel. Needs rope_rows to have run.
msa_status launch_attend_dec_tc(const AttnParams& P, cudaStream_t st);

// attend_dec.cu: the decoding shapes (at most 16 query vectors per tile),
// grid (n_splits, hkv, n_tiles), each split an even share of every
// sequence's memory and local keys; the splits of a (tile, kv head) form one
// cluster. It rotates its own queries and local keys when each CTA's share of
// the local keys is small (otherwise rope_rows rotates both first, with
// krot_split = 1); it lists the routed form's memory rows itself when
// top_k <= kDecRoutedMaxK.
constexpr int kDecMaxSplits = 8;
constexpr int kDecRoutedMaxK = 256;
constexpr int kDecRotKeysMax = 256;  // in-kernel rotation: the local keys of a CTA's first 16 steps at most
msa_status launch_attend_dec(const AttnParams& P, cudaStream_t st);
int attend_dec_error_take();  // 1 if its bounded wait (bulk-copy rows) ran out since the last call
int attend_dec_tc_error_take();

}  // namespace msa
