// Whitened E4M3 codec on the tcgen05 tensor cores (bf16 gradients).
//
// GIFT review page, "What carries the argument": the gradient G of a linear
// layer is whitened on its input side before FP8 quantisation,
//   W = G M,  M = a I + U diag(c) U^T,  a = rho^{-1/2},
//   c_k = (lambda_k + rho)^{-1/2} - a,
// and mapped back with M^{-1} after dequantisation.  Per 128-row panel:
//   E1  P = G U            (M=128, N=64, K=d_in)  tensor cores
//   E2  W = a G + (P o c) U^T  (M=128, N=128 per chunk, K=32)
//   E3  amax per 128-column block, E4M3 codes, fp32 scales
// U is fp32; it is split into bf16 hi + lo parts so that every product is
// exact to ~2^-17 (G is exact in bf16, so E1 needs G.U_hi + G.U_lo; E2 needs
// Pc_hi.U_hi + Pc_lo.U_hi + Pc_hi.U_lo).  Accumulation is fp32 in TMEM.
//
// Data flow (one persistent CTA per SM, 480 threads, warp-specialised):
//   warp 13 lane 0  TMA loads of 128x128 G chunks (two 64-column SW128 boxes)
//                   and of the matching 128 rows of U (fp32)
//   warps 8-11      convert those U rows in place into one bf16 tile
//                   [128 rows][hi 32 | lo 32] with the 128-byte swizzle; the
//                   tile is the MN-major B operand of E1 and the K-major B
//                   operand of E2
//   warp 12         TMEM allocation; one thread issues every MMA
//   warps 0-7       epilogue, two threads per row (TMEM lane quarter warp % 4,
//                   column half warp / 4): form the bf16 hi/lo tile of P o c / a
//                   (the A operand of E2), then per chunk read W / a from TMEM
//                   (G enters it through identity MMAs, so the epilogue reads
//                   no G), find the block maximum (the halves exchange theirs
//                   through shared memory), write the 128 codes of the row into
//                   one of two codes tiles and one scale
//   warp 14 lane 0  TMA store of each chunk's codes tile, then frees the tile
// A stage is freed by the MMA's completion.  A CTA's panels are processed in
// blocks that interleave the second pass of one panel (E2, epilogue-bound, its
// chunks re-read from L2 in reverse order) with the first pass of the next
// (E1, an HBM stream).  Panels of all layers of one launch are assigned on the
// host by longest-first greedy scheduling (a panel costs d_in/128 chunks).
// A launch with few panels runs the CLUSTER instantiation instead: 2 or 4
// CTAs of a thread-block cluster share each panel's chunks and sum their
// partial P through distributed shared memory (see cluster_sum16).  The
// decoder below follows the same plan with its own stages.
#include <algorithm>
#include <queue>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "tma_host.h"

namespace gift {
namespace {

constexpr int kPanel = 128;                 // rows per panel = UMMA M
constexpr int kChunk = 128;                 // columns per step = one scale block
constexpr int kStages = 3;
constexpr int kGBytes = kPanel * kChunk * 2;   // 32 KB: two [128][64] bf16 boxes
constexpr int kGHalf = kGBytes / 2;
constexpr int kUBytes = kChunk * 128;          // 16 KB: [128 rows][64 bf16]
constexpr int kStageBytes = kGBytes + kUBytes;
constexpr int kPcBytes = kPanel * 128;         // 16 KB: [128 rows][64 bf16]
constexpr int kCodesBytes = kPanel * kChunk;    // 16 KB: codes of one chunk
constexpr int kIdBytes = 16 * 128;             // 2 KB: 16 x 16 bf16 identity, 128-byte rows
constexpr int kXBytes = kPanel * 32 * 4;        // 16 KB: fp32 partial projections exchanged in a cluster
// TMEM accumulators of W for the second pass (columns 0..255) and codes
// tiles of the encoder.  A third of either measured no faster on B200.
constexpr int kWBufs = 2, kCBufs = 2;
constexpr int kSmemBytes = kStages * kStageBytes + kPcBytes + kCBufs * kCodesBytes + kIdBytes + 1024 + 512;
constexpr int enc_smem(bool cluster) { return kSmemBytes + (cluster ? kXBytes : 0); }
constexpr int kThreads = 480;  // 8 epilogue + 4 converter + MMA + TMA load + TMA store warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColP = 256;  // two 64-column slots of P: panel parity
constexpr int kLead = 3;         // first-pass steps that open a block (see Steps)
GIFT_DEV uint32_t w_col(int b) { return 128u * (uint32_t)b; }
constexpr uint32_t kIdescE1 = umma_idesc_bf16(128, 64, 0, 1);   // A K-major, B MN-major
constexpr uint32_t kIdescE2 = umma_idesc_bf16(128, 128, 0, 0);  // both K-major
constexpr uint32_t kIdescId = umma_idesc_bf16(128, 16, 0, 0);   // G . I16, both K-major
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kMaxJobs = 48;
constexpr int kMaxPanels = 1536;

struct alignas(64) EncJob {
  CUtensorMap tmG;  // bf16 [d_out][d_in], box [128][64], 128-byte swizzle
  CUtensorMap tmU;  // fp32 U [d_in][32], box [128][32], 128-byte swizzle
  CUtensorMap tmC;  // uint8 codes [d_out][d_in], box [128][128], 128-byte swizzle (E4M3 stores)
  const float* U;
  const float* lambda;
  const float* rho;
  uint8_t* codes;   // E4M3 [d_out][d_in], or NVFP4 [d_out][d_in/2]
  float* scales;    // E4M3 fp32 [d_out][d_in/128]
  uint8_t* sb;      // NVFP4 E4M3 block scales [d_out][d_in/16]
  float* tscale;    // NVFP4 tensor scale (amax bits while encoding)
  int d_out, d_in, rank, fmt;
};

struct EncParams {
  EncJob jobs[kMaxJobs];
  uint16_t sched_off[kNumSMs + 1];  // cluster b runs sched_ids[sched_off[b] .. sched_off[b+1])
  uint16_t sched_ids[kMaxPanels];   // job << 8 | panel
  int split;                        // CTAs per cluster, each taking 1 / split of every panel's chunks
  uint32_t stall_polls;             // test hook (0 = off): see stall_check
  int presplit;                     // 1: tmU maps the caller's U split (no conversion in the kernel)
};
static_assert(sizeof(EncParams) <= 32760, "kernel parameter space");

// 16-byte chunk q of row r of a [rows][128 B] tile with the 128-byte swizzle
GIFT_DEV uint32_t sw128(uint32_t r, uint32_t q) { return r * 128u + ((q ^ (r & 7u)) << 4); }

GIFT_DEV void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// L2 eviction policies for TMA loads: the first pass over a panel keeps its
// chunks (they are read again by the second pass), the second pass lets them go.
GIFT_DEV uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
GIFT_DEV uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
GIFT_DEV void tma_load_2d_hint(uint32_t dst, const void* tmap, uint64_t* bar, int x, int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// 2-D tiled TMA store shared -> global (bulk-group completion).  Rows and
// columns outside the tensor are not written.
GIFT_DEV void tma_store_2d_hint(const void* tmap, uint32_t src, int x, int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group.L2::cache_hint"
      " [%0, {%2, %3}], [%1], %4;" ::"l"(tmap),
      "r"(src), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
GIFT_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed store groups still read shared memory.
template <int N>
GIFT_DEV void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every committed store group has completed.
GIFT_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Walks the steps of one CTA in the order every role uses.  A CTA's panels
// p_0 .. p_{n-1} are visited in blocks: block 0 is the first pass of p_0
// (chunks 0 .. nc-1); block k >= 1 is the second pass of p_{k-1} (chunks
// nc-1 .. 0) interleaved step by step with the first pass of p_k, so that the
// HBM stream of one panel overlaps the epilogue work of the previous one.
// Each block opens with kLead first-pass steps: the second pass of p_{k-1}
// needs P o c of p_{k-1}, which the epilogue forms only once the first pass
// of p_{k-1} has completed, and the MMA issues p_k's first steps meanwhile
// (the encoder keeps P in two TMEM slots, by panel parity).
//
// With a cluster of S CTAs sharing a panel list, CTA rank q runs chunks
// [q nc / S, (q + 1) nc / S) of every panel (nc = d_in / 128 >= S); the step
// counts and the local index below are over that range.
template <class P>
struct Steps {
  const P& p;
  int beg, end, k, q, S;
  int n1, n2, i1, i2;  // first- and second-pass steps of block k, and how many are done
  int pass;            // pass of the current step
  GIFT_DEV Steps(const P& p_, int b, int e, int q_, int s_) : p(p_), beg(b), end(e), k(0), q(q_), S(s_) { setup(); }
  GIFT_DEV int ncg_of(int it) const { return p.jobs[p.sched_ids[it] >> 8].d_in / kChunk; }
  GIFT_DEV int lo_of(int it) const { return (q * ncg_of(it)) / S; }
  GIFT_DEV int nc_of(int it) const { return ((q + 1) * ncg_of(it)) / S - lo_of(it); }
  GIFT_DEV void setup() {
    i1 = i2 = 0;
    n1 = beg + k < end ? nc_of(beg + k) : 0;
    n2 = k >= 1 && beg + k - 1 < end ? nc_of(beg + k - 1) : 0;
    pick();
  }
  GIFT_DEV void pick() { pass = (i2 < n2 && (i1 >= n1 || i1 >= i2 + kLead)) ? 1 : 0; }
  GIFT_DEV bool valid() const { return n1 + n2 > 0; }
  GIFT_DEV int slot() const { return pass ? beg + k - 1 : beg + k; }
  GIFT_DEV int job() const { return p.sched_ids[slot()] >> 8; }
  GIFT_DEV int panel() const { return p.sched_ids[slot()] & 255; }
  GIFT_DEV int nc() const { return pass ? n2 : n1; }                 // this CTA's chunks of the panel
  GIFT_DEV int lidx() const { return pass ? i2 : i1; }                // step index within them
  GIFT_DEV int chunk() const { return lo_of(slot()) + (pass ? n2 - 1 - i2 : i1); }  // chunk of d_in
  GIFT_DEV bool block_start() const { return i1 + i2 == 0; }
  GIFT_DEV void next() {
    if (pass)
      ++i2;
    else
      ++i1;
    if (i1 + i2 == n1 + n2) {
      ++k;
      setup();
    } else {
      pick();
    }
  }
};

// Named barrier that also ORs a predicate over the group: every member gets
// the same answer, so a group can agree to stop without a shared flag.
GIFT_DEV bool named_sync_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %3, 0;\n\t"
      "barrier.red.or.pred p, %1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(n), "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// Test hook of the failure path (stall_polls > 0): before any load or MMA is
// issued, thread 0 waits at most stall_polls polls on `bar`, a barrier that
// nothing arrives at; the wait runs out and sets *failed.  The caller then
// syncs the CTA and every role skips its work, so the kernel returns with
// nothing in flight and reports GIFT_DEV_TIMEOUT.
GIFT_DEV void stall_check(uint32_t stall_polls, uint64_t* bar, int* failed) {
  if (stall_polls && threadIdx.x == 0 && !mbar_wait(bar, 0u, stall_polls)) *failed = 1;
}

GIFT_DEV void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
GIFT_DEV uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// ---- thread-block clusters: the CTAs that split one panel's chunks ----
GIFT_DEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster (kernel start, after the barrier
// inits, and kernel end, so no CTA leaves while a peer may still touch its
// shared memory).
GIFT_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in cluster CTA `rank`.
GIFT_DEV uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
GIFT_DEV void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
GIFT_DEV float4 ld_cluster_v4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}
GIFT_DEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// Sum over the S CTAs of a cluster of one epilogue thread's 16 partial
// projections (row r, coefficients 16 h .. 16 h + 15), added in cluster-rank
// order so that every CTA of the cluster ends with the same fp32 sums.
// xbuf is this CTA's [128][32] fp32 exchange tile; xfull (count 256 (S-1))
// completes when every peer thread has written its partial, xempty (count
// 256 (S-1)) when every peer thread has read this CTA's.  nx counts the
// exchanges so far.  Returns false if a wait ran out.
GIFT_DEV bool cluster_sum16(float (&v)[16], uint32_t xbuf, uint64_t* xfull, uint64_t* xempty, uint32_t& nx, int S,
                            int q, int r, int h) {
  if (nx >= 1 && !mbar_wait_cluster(xempty, (nx - 1) & 1u, kWaitLimit)) return false;
  const uint32_t my = xbuf + (uint32_t)r * 128u + (uint32_t)h * 64u;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    st_shared_v4(my + 16 * i, __float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]), __float_as_uint(v[4 * i + 2]),
                 __float_as_uint(v[4 * i + 3]));
  for (int t = 0; t < S; ++t)
    if (t != q) mbar_arrive_remote(mapa_shared(smem_u32(xfull), t));
  if (!mbar_wait_cluster(xfull, nx & 1u, kWaitLimit)) return false;
  float sum[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) sum[k] = 0.0f;
  for (int t = 0; t < S; ++t) {
    const uint32_t src = mapa_shared(my, t);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 w = ld_cluster_v4(src + 16 * i);
      sum[4 * i] += w.x;
      sum[4 * i + 1] += w.y;
      sum[4 * i + 2] += w.z;
      sum[4 * i + 3] += w.w;
    }
  }
  for (int t = 0; t < S; ++t)
    if (t != q) mbar_arrive_remote(mapa_shared(smem_u32(xempty), t));
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = sum[k];
  ++nx;
  return true;
}


// Split fp32 into bf16 hi (RNE) and bf16 lo = RNE(x - hi).
GIFT_DEV void split_bf16(float x, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  lo = x - hi;
}

// bf16 split [hi 0..31 | lo 0..31] of a U row into row t of a [128][128 B]
// tile with the 128-byte swizzle.
GIFT_DEV void store_u_split_bf16(uint32_t tile, int t, const float (&u)[32]) {
  uint32_t hi[16], lo[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float h0, l0, h1, l1;
    split_bf16(u[2 * k], h0, l0);
    split_bf16(u[2 * k + 1], h1, l1);
    hi[k] = pack_bf16x2(h0, h1);
    lo[k] = pack_bf16x2(l0, l1);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) st_shared_v4(tile + sw128(t, q), hi[4 * q], hi[4 * q + 1], hi[4 * q + 2], hi[4 * q + 3]);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    st_shared_v4(tile + sw128(t, 4 + q), lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
}

// As store_u_split_bf16, with f16 parts for the decoder's first pass:
// [hi 0..31 | lo 0..31] with hi = f16(u) and lo = f16((u - hi) * 2^11) (the
// product with lo is scaled back by 2^-11 in the epilogue).  f16 keeps 11
// mantissa bits per part, and every E4M3 or NVFP4 value is exact in f16.
constexpr float kF16LoScale = 2048.0f;
GIFT_DEV void store_u_split_f16(uint32_t tile, int t, const float (&u)[32]) {
  uint32_t hi[16], lo[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float h0 = __half2float(__float2half_rn(u[2 * k]));
    const float h1 = __half2float(__float2half_rn(u[2 * k + 1]));
    hi[k] = pack_f16x2(h0, h1);
    lo[k] = pack_f16x2((u[2 * k] - h0) * kF16LoScale, (u[2 * k + 1] - h1) * kF16LoScale);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) st_shared_v4(tile + sw128(t, q), hi[4 * q], hi[4 * q + 1], hi[4 * q + 2], hi[4 * q + 3]);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    st_shared_v4(tile + sw128(t, 4 + q), lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
}

// Row t of a U tile that TMA placed in shared memory as fp32 (one 128-byte
// swizzled row), or row `row` of U read from global memory (L2-resident).
GIFT_DEV void u_row_from_tile(uint32_t tile, int t, float (&u)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint4 v = ld_shared_v4(tile + sw128(t, q));
    u[4 * q] = __uint_as_float(v.x);
    u[4 * q + 1] = __uint_as_float(v.y);
    u[4 * q + 2] = __uint_as_float(v.z);
    u[4 * q + 3] = __uint_as_float(v.w);
  }
}
// The transform's coefficients of the layer of schedule entry `it`, written by
// one warp into a shared-memory slot of 33 floats: c_k / a = (rho / (lambda_k +
// rho))^{1/2} - 1 for k < rank (0 beyond), then a = rho^{-1/2}.  Formed once per
// panel, a block ahead of their use, off the path of the MMA's wait for P o c.
GIFT_DEV void enc_coefs(const EncParams& p, int it, float* slot, int lane) {
  const EncJob& J = p.jobs[p.sched_ids[it] >> 8];
  const double rho = (double)__ldg(J.rho);
  slot[lane] = lane < J.rank ? (float)(sqrt(rho / ((double)__ldg(J.lambda + lane) + rho)) - 1.0) : 0.0f;
  if (lane == 0) slot[32] = (float)(1.0 / sqrt(rho));
}

template <int FMT, bool CLUSTER>
__global__ void __launch_bounds__(kThreads, 1) whiten_encode_tc_kernel(const __grid_constant__ EncParams p,
                                                                     uint32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t pc_tile = sbase + kStages * kStageBytes;
  const uint32_t cbuf = pc_tile + kPcBytes;             // [2] codes tiles [128][128 B], 128-byte swizzle
  const uint32_t id_tile = cbuf + kCBufs * kCodesBytes;  // 16 x 16 identity, K-major, 128-byte swizzle
  const uint32_t xbuf = id_tile + kIdBytes;             // [128][32] fp32 partial P (CLUSTER only)
  uint64_t* bars = (uint64_t*)(smem + kStages * kStageBytes + kPcBytes + kCBufs * kCodesBytes + kIdBytes +
                               (CLUSTER ? kXBytes : 0));
  uint64_t* full = bars;                  // [kStages] count 1: converter (stage ready for the MMA)
  uint64_t* empty = bars + kStages;       // [kStages] count 1: MMA commit
  uint64_t* tfull = bars + 2 * kStages;   // [kStages] count 1 + tx: TMA (G and fp32 U)
  uint64_t* p_full = bars + 3 * kStages;  // [2: p_full, p_full + 17] count 1 (MMA commit): P of a panel, by parity
  uint64_t* pc_full = p_full + 1;         // count 256 (epilogue)
  uint64_t* w_full = p_full + 2;          // [kWBufs] count 1
  uint64_t* w_empty = p_full + 5;         // [kWBufs] count 256
  uint64_t* cready = p_full + 8;          // [kCBufs] count 256: a codes tile is written
  uint64_t* cfree = p_full + 11;          // [kCBufs] count 1: the store of a codes tile has read it
  uint64_t* xfull = p_full + 14;          // count 256 (S-1): the peers' partials are written (clusters)
  uint64_t* xempty = p_full + 15;         // count 256 (S-1): the peers have read this CTA's partial
  uint64_t* stall = p_full + 16;          // count 1, never arrived at (test hook)
  uint32_t* tmem_slot = (uint32_t*)(p_full + 18);
  __shared__ int failed;  // any role gave up (reported at exit)
  __shared__ int nonfin;  // a block maximum was not finite (reported at exit)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = CLUSTER ? p.split : 1;  // without clusters, the split arithmetic folds away
  const int q = CLUSTER ? (int)cluster_ctarank() : 0;
  const int beg = p.sched_off[blockIdx.x / S], end = p.sched_off[blockIdx.x / S + 1];

  if (threadIdx.x == 0) {
    failed = 0;
    nonfin = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&tfull[s], 1);
    }
    mbar_init(p_full, 1);
    mbar_init(p_full + 17, 1);
    mbar_init(pc_full, 256);
    mbar_init(stall, 1);
    for (int b = 0; b < 3; ++b) {
      mbar_init(&w_full[b], 1);
      mbar_init(&w_empty[b], 256);
      mbar_init(&cready[b], 256);
      mbar_init(&cfree[b], 1);
    }
    if (CLUSTER) {
      mbar_init(xfull, 256 * (S - 1));
      mbar_init(xempty, 256 * (S - 1));
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    // identity I16 as a K-major B operand: row n holds e_n in its first 32 bytes
    for (int n = lane; n < 16; n += 32) {
#pragma unroll
      for (int q = 0; q < 8; ++q) st_shared_v4(id_tile + sw128(n, q), 0u, 0u, 0u, 0u);
      const uint32_t one = 0x3F80u << (16 * (n & 1));  // bf16 1.0 in the half of the word for column n
      const uint32_t w4[4] = {(n & 7) >> 1 == 0 ? one : 0u, (n & 7) >> 1 == 1 ? one : 0u,
                              (n & 7) >> 1 == 2 ? one : 0u, (n & 7) >> 1 == 3 ? one : 0u};
      st_shared_v4(id_tile + sw128(n, n >> 3), w4[0], w4[1], w4[2], w4[3]);
    }
    fence_async_shared();
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (CLUSTER) cluster_sync_all();  // the peers' barriers are initialised before any remote arrive
  const uint32_t tbase = *tmem_slot;
  stall_check(p.stall_polls, stall, &failed);
  __syncthreads();
  const bool skip = failed != 0;  // the same for every thread: read after the barrier

  if (skip) {
    // the test hook's wait ran out: nothing was issued, nothing to do
  } else if (warp == 13) {
    // ---------------- TMA producer: G chunks and U rows, running ahead of the ring ----------------
    if (lane == 0) {
      const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
      uint32_t step = 0;
      for (Steps<EncParams> st(p, beg, end, q, S); st.valid() && !failed; st.next(), ++step) {
        const int s = step % kStages;
        const uint32_t use = step / kStages;
        if (step >= kStages && !mbar_wait(&empty[s], (use - 1) & 1u, kWaitLimit)) {
          failed = 1;
          break;
        }
        const EncJob& J = p.jobs[st.job()];
        const uint64_t pol = st.pass == 0 ? keep : drop;
        const uint32_t dst = sbase + s * kStageBytes;
        mbar_arrive_expect_tx(&tfull[s], kGBytes + kUBytes);
        tma_load_2d_hint(dst, &J.tmG, &tfull[s], st.chunk() * kChunk, st.panel() * kPanel, pol);
        tma_load_2d_hint(dst + kGHalf, &J.tmG, &tfull[s], st.chunk() * kChunk + 64, st.panel() * kPanel, pol);
        // U: fp32 rows (split by the converters), or the caller's bf16 [hi | lo] rows
        tma_load_2d_hint(dst + kGBytes, &J.tmU, &tfull[s], 0, st.chunk() * kChunk, keep);
      }
    }
  } else if (warp == 14) {
    // ---------------- code stores: one TMA store per second-pass step ----------------
    if (lane == 0) {
      const uint64_t drop = policy_evict_first();
      uint32_t e2 = 0;
      for (Steps<EncParams> st(p, beg, end, q, S); st.valid() && !failed; st.next()) {
        if (st.pass == 0) continue;
        const int cb = (int)(e2 % kCBufs);
        if (!mbar_wait(&cready[cb], (e2 / kCBufs) & 1u, kWaitLimit)) {
          failed = 1;
          break;
        }
        const EncJob& J = p.jobs[st.job()];
        if (FMT == kFmtE4M3) {  // NVFP4 codes were stored by the epilogue
          tma_store_2d_hint(&J.tmC, cbuf + cb * kCodesBytes, st.chunk() * kChunk, st.panel() * kPanel, drop);
          bulk_commit();
          bulk_wait_read<0>();
        }
        mbar_arrive(&cfree[cb]);
        ++e2;
      }
      bulk_wait_all();
    }
  } else if (warp >= 8 && warp < 12) {
    // ---------------- converters: fp32 U rows -> bf16 hi/lo, in place, one row each ----------------
    // Exit decisions are voted at a named barrier so all 128 threads leave
    // at the same step.
    const int t = threadIdx.x - 256;
    uint32_t step = 0;
    // with a pre-split U the stages are ready as TMA lands them: nothing to do
    for (Steps<EncParams> st(p, beg, end, q, S); st.valid() && !p.presplit; st.next(), ++step) {
      const int s = step % kStages;
      const uint32_t use = step / kStages;
      float u[32];
      const bool ok = mbar_wait(&tfull[s], use & 1u, kWaitLimit);
      if (named_sync_or(1, 128, !ok)) {
        failed = 1;
        break;
      }
      const uint32_t u_tile = sbase + s * kStageBytes + kGBytes;
      u_row_from_tile(u_tile, t, u);
      store_u_split_bf16(u_tile, t, u);
      fence_async_shared();
      named_sync(1, 128);
      if (t == 0) mbar_arrive(&full[s]);
    }
  } else if (warp == 12) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t step = 0, e2 = 0;
      for (Steps<EncParams> st(p, beg, end, q, S); st.valid() && !failed; st.next(), ++step) {
        const int s = step % kStages;
        // the second pass of p_{k-1} needs its P o (c/a) in shared memory; that
        // also means P of p_{k-1} has been read from its TMEM slot, which the
        // first pass of p_{k+1} reuses
        if (st.pass == 1 && st.i2 == 0 && !mbar_wait(pc_full, (st.k - 1) & 1u, kWaitLimit)) { failed = 1; break; }
        if (!mbar_wait(p.presplit ? &tfull[s] : &full[s], (step / kStages) & 1u, kWaitLimit)) { failed = 1; break; }
        tc_fence_after();
        const uint32_t g_tile = sbase + s * kStageBytes, u_tile = g_tile + kGBytes;
        if (st.pass == 0) {
          // E1: P2[128 x 64] += G_c . [U_hi | U_lo]_c over this CTA's chunks
          const int c = st.lidx();
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = umma_desc_sw128(g_tile + h * kGHalf + kk * 32, 16, 1024);
              const uint64_t bd = umma_desc_sw128(u_tile + (h * 64 + kk * 16) * 128, 16, 1024);
              umma_bf16(tbase + kColP + 64u * (st.k & 1), ad, bd, kIdescE1, (c | h | kk) ? 1u : 0u);
            }
          umma_commit(&empty[s]);
          // one barrier per panel parity: the first pass of p_{k+1} may complete
          // before the epilogue has waited for p_k's
          if (c == st.nc() - 1) umma_commit((st.k & 1) ? p_full + 17 : p_full);
        } else {
          // E2: W/a [128 x 128] = Pc_hi U_hi^T + Pc_lo U_hi^T + Pc_hi U_lo^T + G . I
          // (Pc already divided by a; G . I adds G exactly, 16 columns per MMA)
          const int b = (int)(e2 % kWBufs);
          if (e2 >= kWBufs && !mbar_wait(&w_empty[b], ((e2 / kWBufs) - 1) & 1u, kWaitLimit)) { failed = 1; break; }
          tc_fence_after();
          const uint32_t d = tbase + w_col(b);
          const int ak[6] = {0, 16, 32, 48, 0, 16};   // Pc: hi = k 0..31, lo = k 32..63
          const int bk[6] = {0, 16, 0, 16, 32, 48};   // U : hi = k 0..31, lo = k 32..63
#pragma unroll
          for (int q = 0; q < 6; ++q) {
            const uint64_t ad = umma_desc_sw128(pc_tile + ak[q] * 2, 16, 1024);
            const uint64_t bd = umma_desc_sw128(u_tile + bk[q] * 2, 16, 1024);
            umma_bf16(d, ad, bd, kIdescE2, q ? 1u : 0u);
          }
          const uint64_t idd = umma_desc_sw128(id_tile, 16, 1024);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint64_t ad = umma_desc_sw128(g_tile + (j >> 2) * kGHalf + (j & 3) * 32, 16, 1024);
            umma_bf16(d + 16 * j, ad, idd, kIdescId, 1u);
          }
          umma_commit(&empty[s]);
          umma_commit(&w_full[b]);
          ++e2;
        }
      }
    }
  } else {
    // ---------------- epilogue: warps 0-7 ----------------
    // Thread (r, h): row r = 32 (warp % 4) + lane of the panel (its TMEM
    // lane), columns 64 h .. 64 h + 63 of every 128-column chunk (h = warp / 4).
    // TMEM holds W' = W / a; the two halves of a row exchange their partial
    // block maxima through shared memory and write their codes into one of two
    // codes tiles for the store warp.
    __shared__ float amax_x[2][128];
    __shared__ float coefs[2][33];  // by panel parity: see enc_coefs
    const int h = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    if (warp == 0 && beg < end) enc_coefs(p, beg, coefs[0], lane);  // p_0 (read after a barrier)
    uint32_t e2 = 0, nx = 0;
    float a = 0.0f;
    float S_t = 0.0f;   // NVFP4 tensor scale (codes pass)
    float pmax = 0.0f;  // NVFP4 amax pass: this thread's max |W'| over the panel
    bool stop = false;  // group vote: set for all 256 threads at the same barrier
    for (Steps<EncParams> st(p, beg, end, q, S); st.valid() && !stop; st.next()) {
      if (st.pass == 0) continue;  // first-pass steps are the MMA's alone
      const EncJob& J = p.jobs[st.job()];
      const int panel = st.panel();
      if (st.i2 == 0) {
        if (FMT == kFmtNvfp4) S_t = nvfp4_tensor_scale(__uint_as_float(*reinterpret_cast<volatile uint32_t*>(J.tscale)));
        // P o (c / a) of this panel for k = 16 h .. 16 h + 15, split into the bf16
        // A operand of E2 (coefficients from the panel's slot, formed a block ago)
        stop = named_sync_or(2, 256, !mbar_wait(((st.k - 1) & 1) ? p_full + 17 : p_full, ((st.k - 1) >> 1) & 1u,
                                                kWaitLimit));
        if (stop) {
          failed = 1;
          break;
        }
        const float* cs = coefs[(st.k - 1) & 1];
        a = cs[32];
        float cf[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) cf[k] = cs[16 * h + k];
        tc_fence_after();
        uint32_t ph[16], pl[16];
        const uint32_t pcol = kColP + 64u * ((st.k - 1) & 1);  // P of p_{k-1}
        tmem_ld16(tbase + lane_off + pcol + 16 * h, ph);
        tmem_ld16(tbase + lane_off + pcol + 32 + 16 * h, pl);
        tmem_wait_ld();
        float pv[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) pv[k] = __uint_as_float(ph[k]) + __uint_as_float(pl[k]);
        if (CLUSTER) {
          // this CTA's chunks gave a partial P: the cluster sums the partials
          stop = named_sync_or(2, 256, !cluster_sum16(pv, xbuf, xfull, xempty, nx, S, q, r, h));
          if (stop) {
            failed = 1;
            break;
          }
        }
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float v0 = pv[2 * k] * cf[2 * k];
          const float v1 = pv[2 * k + 1] * cf[2 * k + 1];
          float h0, l0, h1, l1;
          split_bf16(v0, h0, l0);
          split_bf16(v1, h1, l1);
          hi[k] = pack_bf16x2(h0, h1);
          lo[k] = pack_bf16x2(l0, l1);
        }
        st_shared_v4(pc_tile + sw128(r, 2 * h), hi[0], hi[1], hi[2], hi[3]);
        st_shared_v4(pc_tile + sw128(r, 2 * h + 1), hi[4], hi[5], hi[6], hi[7]);
        st_shared_v4(pc_tile + sw128(r, 4 + 2 * h), lo[0], lo[1], lo[2], lo[3]);
        st_shared_v4(pc_tile + sw128(r, 5 + 2 * h), lo[4], lo[5], lo[6], lo[7]);
        fence_async_shared();
        tc_fence_before();
        mbar_arrive(pc_full);
        // the next panel's coefficients (its slot was last read a block ago)
        if (warp == 0 && beg + st.k < end) enc_coefs(p, beg + st.k, coefs[st.k & 1], lane);
      }
      const int c = st.chunk();
      const int b = (int)(e2 % kWBufs);
      const int64_t row = (int64_t)panel * kPanel + r;
      const bool live = row < J.d_out;
      stop = named_sync_or(2, 256, !mbar_wait(&w_full[b], (e2 / kWBufs) & 1u, kWaitLimit));
      if (stop) {
        failed = 1;
        break;
      }
      tc_fence_after();
      const uint32_t wcol = tbase + lane_off + w_col(b) + 64 * h;
      uint32_t w[64];
      tmem_ld32(wcol, w);
      tmem_ld32(wcol + 32, w + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&w_empty[b]);
      float m0 = 0.0f, m1 = 0.0f, m2 = 0.0f, m3 = 0.0f;
#pragma unroll
      for (int k = 0; k < 64; k += 4) {
        m0 = fmax_nan(m0, fabsf(__uint_as_float(w[k])));
        m1 = fmax_nan(m1, fabsf(__uint_as_float(w[k + 1])));
        m2 = fmax_nan(m2, fabsf(__uint_as_float(w[k + 2])));
        m3 = fmax_nan(m3, fabsf(__uint_as_float(w[k + 3])));
      }
      amax_x[h][r] = fmax_nan(fmax_nan(m0, m1), fmax_nan(m2, m3));
      if (FMT == kFmtNvfp4Amax) {
        // amax(W) = a max|W'| (rounded once); one atomic per warp at the panel's end
        pmax = fmaxf(pmax, live ? amax_x[h][r] : 0.0f);
        if (st.i2 == st.nc() - 1) {
          const float wm = warp_max(pmax);
          if (lane == 0 && wm > 0.0f) atomicMax(reinterpret_cast<uint32_t*>(J.tscale), __float_as_uint(__fmul_rn(a, wm)));
          pmax = 0.0f;
        }
      } else if (FMT == kFmtNvfp4 && live) {
        // four NVFP4 blocks of 16 from W = a W'
        uint2 c4[4];
        uint32_t sbw = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(a, __uint_as_float(w[16 * j + i]));
          uint8_t sbj;
          c4[j] = nvfp4_block16(v, S_t, &sbj);
          sbw |= (uint32_t)sbj << (8 * j);
        }
        uint4* cd = reinterpret_cast<uint4*>(J.codes + row * (J.d_in / 2) + st.chunk() * 64 + 32 * h);
        cd[0] = make_uint4(c4[0].x, c4[0].y, c4[1].x, c4[1].y);
        cd[1] = make_uint4(c4[2].x, c4[2].y, c4[3].x, c4[3].y);
        *reinterpret_cast<uint32_t*>(J.sb + row * (J.d_in / 16) + st.chunk() * 8 + 4 * h) = sbw;
      }
      // the codes tile is free once the store of its previous use has read it;
      // this barrier also exchanges the halves' maxima
      const int cb = (int)(e2 % kCBufs);
      const bool freed = e2 < (uint32_t)kCBufs || mbar_wait(&cfree[cb], ((e2 / kCBufs) - 1) & 1u, kWaitLimit);
      stop = named_sync_or(2, 256, !freed);
      if (stop) {
        failed = 1;
        break;
      }
      // block maximum of W = a W' (rounded once), then the codes of W' x (a 448 / amax)
      const float amax = __fmul_rn(a, fmax_nan(amax_x[0][r], amax_x[1][r]));
      if (live && h == 0 && not_finite(amax)) nonfin = 1;
      const float inv = e4m3_inv_scale(amax);
      const float ai = __fmul_rn(a, inv);
      uint32_t cw[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const uint32_t c01 = f32x2_to_e4m3x2(__fmul_rn(__uint_as_float(w[4 * q]), ai),
                                             __fmul_rn(__uint_as_float(w[4 * q + 1]), ai));
        const uint32_t c23 = f32x2_to_e4m3x2(__fmul_rn(__uint_as_float(w[4 * q + 2]), ai),
                                             __fmul_rn(__uint_as_float(w[4 * q + 3]), ai));
        cw[q] = inv > 0.0f ? (c01 | (c23 << 16)) : 0u;
      }
      if (FMT == kFmtE4M3 && live && h == 0) J.scales[row * (J.d_in / kChunk) + c] = e4m3_scale(amax, inv);
      const uint32_t c_tile = cbuf + cb * kCodesBytes;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_shared_v4(c_tile + sw128(r, 4 * h + q), cw[4 * q], cw[4 * q + 1], cw[4 * q + 2], cw[4 * q + 3]);
      fence_async_shared();
      mbar_arrive(&cready[cb]);
      ++e2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CLUSTER) cluster_sync_all();
  if (warp == 12) tmem_dealloc(tbase, kTmemCols);
  if (threadIdx.x == 0 && err && (failed || nonfin))
    atomicOr(err, (failed ? GIFT_DEV_TIMEOUT : 0u) | (nonfin ? GIFT_DEV_NONFINITE : 0u));
}

// ===========================================================================
// Decode: G_hat = W_hat M^{-1},  W_hat = value(codes) * scale (per block),
//   M^{-1} = a I + U diag(c) U^T,  a = rho^{1/2},  c_k = (lambda_k+rho)^{1/2} - a.
//   D2  P = W_hat U = sum_c s_c (q_c U_c): the codes q are exact in f16, so
//       each chunk's product T_c = q_c [U_hi | U_lo 2^11] (f16 operands, M=128,
//       N=64, K=128) is scaled by its block scale in the epilogue and summed in
//       fp32 (f16 widening is one instruction per pair of codes).
//   D3  G_hat = a W_hat + (P o c) U^T   (M=128, N=128 per chunk, K=32, bf16
//       split as in the encoder), bf16 output with round-to-nearest-even.
// Stage (ring of kDStages) = codes tile (TMA, [128][128 B], 128-byte swizzle)
// + U tile (split to f16 for D2, to bf16 for D3).  D2's A operand, the step's
// codes widened to f16, lives in TMEM: the converter warps write it with
// tcgen05.st into one of two 64-column tiles (row r in lane r), freed when
// the MMA that read it completes.  D3's bf16 output goes through kDOut
// shared-memory tiles, written by the epilogue and freed once the TMA stores
// have read them.  A first-pass stage is released by the D2 commit; a
// second-pass stage as soon as every epilogue thread holds its codes in
// registers (D3, which reads the stage's U, has completed by then).
// ===========================================================================
constexpr int kDStages = 4;                         // decode ring
constexpr int kDOut = 2;                            // output tiles
constexpr int kDCodes = kPanel * kChunk;            // 16 KB
constexpr int kDStageBytes = kDCodes + kUBytes;     // codes + U
constexpr int kDOutBytes = kPanel * kChunk * 2;     // 32 KB: two [128][64] bf16 boxes
constexpr int kDSmemBytes = kDStages * kDStageBytes + kDOut * kDOutBytes + kPcBytes + 1024 + 512;
constexpr int dec_smem(bool cluster) { return kDSmemBytes + (cluster ? kXBytes : 0); }
static_assert(dec_smem(true) <= 232448, "decode shared memory");
static_assert(enc_smem(true) <= 232448, "encode shared memory");
constexpr uint32_t kColT0 = 256, kColT1 = 320;  // D2 accumulators (D3's are w_col(0), w_col(1))
constexpr uint32_t kColA = 384;                 // two 64-column D2 A tiles: 128 f16 codes per lane
constexpr uint32_t kIdescD2 = umma_idesc_f16(128, 64, 0, 1);   // D2 runs on f16 operands

struct alignas(64) DecJob {
  CUtensorMap tmC;  // uint8 codes [d_out][d_in], box [128][128], 128-byte swizzle
  CUtensorMap tmU;  // fp32 U [d_in][32], box [128][32], 128-byte swizzle
  CUtensorMap tmO;  // bf16 G_hat [d_out][d_in], box [128][64], 128-byte swizzle (stores)
  const float* U;
  const float* lambda;
  const float* rho;
  const float* scales;    // E4M3 fp32 [d_out][d_in/128]
  const uint8_t* codes;   // NVFP4 [d_out][d_in/2] (read directly; E4M3 codes arrive by TMA)
  const uint8_t* sb;      // NVFP4 E4M3 block scales [d_out][d_in/16]
  const float* tscale;    // NVFP4 tensor scale
  int d_out, d_in, rank, fmt;
};

struct DecParams {
  DecJob jobs[kMaxJobs];
  uint16_t sched_off[kNumSMs + 1];  // cluster b runs sched_ids[sched_off[b] .. sched_off[b+1])
  uint16_t sched_ids[kMaxPanels];   // job << 8 | panel
  int split;                        // CTAs per cluster, each taking 1 / split of every panel's chunks
  uint32_t stall_polls;             // test hook (0 = off): see stall_check
  int presplit;                     // 1: tmU maps the caller's U split (no conversion in the kernel)
};
static_assert(sizeof(DecParams) <= 32760, "kernel parameter space");

// E4M3 pair -> f16 pair (exact: every E4M3 value is an f16 value), byte 0 in the low half
GIFT_DEV uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  return h;
}

// As enc_coefs, for the inverse: c'_k = (lambda_k + rho)^{1/2} - rho^{1/2} for
// k < rank (0 beyond), then a = rho^{1/2}.
GIFT_DEV void dec_coefs(const DecParams& p, int it, float* slot, int lane) {
  const DecJob& J = p.jobs[p.sched_ids[it] >> 8];
  const double rho = (double)__ldg(J.rho);
  const double a64 = sqrt(rho);
  slot[lane] = lane < J.rank ? (float)(sqrt((double)__ldg(J.lambda + lane) + rho) - a64) : 0.0f;
  if (lane == 0) slot[32] = (float)a64;
}

template <int FMT, bool CLUSTER>
__global__ void __launch_bounds__(kThreads, 1) whiten_decode_tc_kernel(const __grid_constant__ DecParams p,
                                                                     uint32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t otile = sbase + kDStages * kDStageBytes;  // [kDOut] output tiles: two [128][64] bf16 boxes each
  const uint32_t pc_tile = otile + kDOut * kDOutBytes;
  const uint32_t xbuf = pc_tile + kPcBytes;  // [128][32] fp32 partial P (CLUSTER only)
  uint64_t* bars = (uint64_t*)(smem + kDStages * kDStageBytes + kDOut * kDOutBytes + kPcBytes + (CLUSTER ? kXBytes : 0));
  uint64_t* full = bars;                   // [kDStages] count 1: converter (U split; first pass: A tile written)
  uint64_t* cfull = bars + kDStages;       // [kDStages] count 1 + tx: TMA (codes and U)
  uint64_t* empty = bars + 2 * kDStages;   // [kDStages] count 1: MMA commit (D2) or epilogue (D3, codes read)
  uint64_t* afree = bars + 3 * kDStages;   // [2] count 1: TMEM A tile free (MMA commit)
  uint64_t* ofree = afree + 2;             // [kDOut <= 2] count 1: output tile stored (store warp)
  uint64_t* oready = ofree + 2;            // [kDOut <= 2] count 256: output tile written
  uint64_t* t_full = oready + 2;           // [2] count 1
  uint64_t* t_empty = t_full + 2;          // [2] count 256
  uint64_t* pc_full = t_full + 4;          // count 256
  uint64_t* w_full = t_full + 5;           // [kWBufs] count 1
  uint64_t* w_empty = t_full + 8;          // [kWBufs] count 256
  uint64_t* xfull = t_full + 11;           // count 256 (S-1): the peers' partials are written (clusters)
  uint64_t* xempty = t_full + 12;          // count 256 (S-1): the peers have read this CTA's partial
  uint64_t* stall = t_full + 13;           // count 1, never arrived at (test hook)
  uint32_t* tmem_slot = (uint32_t*)(t_full + 14);
  __shared__ int failed;
  __shared__ int nonfin;  // a block scale was not finite (reported at exit)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = CLUSTER ? p.split : 1;  // without clusters, the split arithmetic folds away
  const int q = CLUSTER ? (int)cluster_ctarank() : 0;
  const int beg = p.sched_off[blockIdx.x / S], end = p.sched_off[blockIdx.x / S + 1];
  if (threadIdx.x == 0) {
    failed = 0;
    nonfin = 0;
    mbar_init(stall, 1);
    for (int s = 0; s < kDStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&cfull[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afree[b], 1);
      mbar_init(&t_full[b], 1);
      mbar_init(&t_empty[b], 256);
    }
    for (int o = 0; o < kDOut; ++o) {
      mbar_init(&ofree[o], 1);
      mbar_init(&oready[o], 256);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&w_full[b], 1);
      mbar_init(&w_empty[b], 256);
    }
    mbar_init(pc_full, 256);
    if (CLUSTER) {
      mbar_init(xfull, 256 * (S - 1));
      mbar_init(xempty, 256 * (S - 1));
    }
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (CLUSTER) cluster_sync_all();  // the peers' barriers are initialised before any remote arrive
  const uint32_t tbase = *tmem_slot;
  stall_check(p.stall_polls, stall, &failed);
  __syncthreads();
  const bool skip = failed != 0;  // the same for every thread: read after the barrier

  if (skip) {
    // the test hook's wait ran out: nothing was issued, nothing to do
  } else if (warp == 13) {
    // ---------------- TMA producer: codes chunks and U rows, running ahead of the ring ----------------
    if (lane == 0) {
      const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
      uint32_t step = 0;
      for (Steps<DecParams> st(p, beg, end, q, S); st.valid() && !failed; st.next(), ++step) {
        const int s = step % kDStages;
        const uint32_t use = step / kDStages;
        if (step >= kDStages && !mbar_wait(&empty[s], (use - 1) & 1u, kWaitLimit)) {
          failed = 1;
          break;
        }
        const DecJob& J = p.jobs[st.job()];
        const uint32_t dst = sbase + s * kDStageBytes;
        const uint32_t ub = (uint32_t)kUBytes;
        if (FMT == kFmtE4M3) {
          mbar_arrive_expect_tx(&cfull[s], kDCodes + ub);
          tma_load_2d_hint(dst, &J.tmC, &cfull[s], st.chunk() * kChunk, st.panel() * kPanel,
                           st.pass == 0 ? keep : drop);
        } else {
          mbar_arrive_expect_tx(&cfull[s], ub);  // NVFP4 codes are read from global memory
        }
        // U: fp32 rows (split by the converters), or the caller's split, whose rows
        // d_in .. 2 d_in - 1 hold the f16 parts for D2 and rows 0 .. d_in - 1 the
        // bf16 parts for D3
        const int urow = (p.presplit && st.pass == 0 ? J.d_in : 0) + st.chunk() * kChunk;
        tma_load_2d_hint(dst + kDCodes, &J.tmU, &cfull[s], 0, urow, keep);
      }
    }
  } else if (warp == 14) {
    // ---------------- output stores: a second-pass step's tile leaves by two TMA stores ----------------
    if (lane == 0) {
      const uint64_t drop = policy_evict_first();
      uint32_t e2 = 0;  // second-pass steps so far
      for (Steps<DecParams> st(p, beg, end, q, S); st.valid() && !failed; st.next()) {
        if (st.pass == 0) continue;
        const int o = (int)(e2 % kDOut);
        if (!mbar_wait(&oready[o], (e2 / kDOut) & 1u, kWaitLimit)) {
          failed = 1;
          break;
        }
        const DecJob& J = p.jobs[st.job()];
        const uint32_t o_tile = otile + o * kDOutBytes;
        tma_store_2d_hint(&J.tmO, o_tile, st.chunk() * kChunk, st.panel() * kPanel, drop);
        tma_store_2d_hint(&J.tmO, o_tile + kGHalf, st.chunk() * kChunk + 64, st.panel() * kPanel, drop);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(&ofree[o]);
        ++e2;
      }
      bulk_wait_all();
    }
  } else if (warp >= 8 && warp < 12) {
    // ---------------- converters: U split in place; first pass: codes widened into a TMEM A tile ----------------
    // With a pre-split U, first-pass stages need only the codes widened and
    // second-pass stages nothing; the converters still take every stage in
    // turn, so their waits on the stages never fall a phase behind the ring
    // (a stage is reloaded only after the MMA has taken it, and the MMA
    // takes it after the converters).
    const int t = threadIdx.x - 256;  // row t = TMEM lane t (warps 8-11 own lane quarters 0-3)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t step = 0, d2 = 0;
    for (Steps<DecParams> st(p, beg, end, q, S); st.valid(); st.next(), ++step) {
      const int s = step % kDStages, a = d2 & 1;
      const uint32_t use = step / kDStages;
      float u[32];
      bool ok = mbar_wait(&cfull[s], use & 1u, kWaitLimit);
      if (st.pass == 0 && d2 >= 2) ok = ok && mbar_wait(&afree[a], ((d2 >> 1) - 1) & 1u, kWaitLimit);
      if (named_sync_or(1, 128, !ok)) {
        failed = 1;
        break;
      }
      tc_fence_after();  // the MMA that read A tile a has completed
      const uint32_t c_tile = sbase + s * kDStageBytes;
      const uint32_t u_tile = c_tile + kDCodes;
      const uint32_t a_tile = tbase + lane_off + kColA + 64u * (uint32_t)a;  // columns: f16 pairs of row t
      // D2 multiplies f16 codes by an f16 split of U, D3 the bf16 P' o c' by a bf16 split
      if (!p.presplit) {
        u_row_from_tile(u_tile, t, u);
        if (st.pass == 0)
          store_u_split_f16(u_tile, t, u);
        else
          store_u_split_bf16(u_tile, t, u);
      }
      const DecJob& J = p.jobs[st.job()];
      if (st.pass == 0 && FMT != kFmtE4M3) {
        // NVFP4: row t's 128 codes (64 bytes) and 8 block scales from global,
        // widened to f16 value(code) x value(scale) (exact)
        const int64_t row = (int64_t)st.panel() * kPanel + t;
        uint4 cw[4] = {};
        uint2 sw = make_uint2(0u, 0u);
        if (row < J.d_out) {
          const uint4* src = reinterpret_cast<const uint4*>(J.codes + row * (J.d_in / 2) + st.chunk() * 64);
#pragma unroll
          for (int q = 0; q < 4; ++q) cw[q] = __ldg(src + q);
          sw = __ldg(reinterpret_cast<const uint2*>(J.sb + row * (J.d_in / 16) + st.chunk() * 8));
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {  // block b = columns 16 b .. 16 b + 15
          const uint4& c = cw[b >> 1];
          const uint2 cb = (b & 1) ? make_uint2(c.z, c.w) : make_uint2(c.x, c.y);
          float v[16];
          nvfp4_block16_values(cb, (uint8_t)(((b < 4) ? sw.x : sw.y) >> (8 * (b & 3))), v);
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = pack_f16x2(v[2 * i], v[2 * i + 1]);
          tmem_st8(a_tile + 8u * b, o);  // columns 16 b .. 16 b + 15 of the chunk
        }
      } else if (st.pass == 0) {
        // the codes of row t, widened to f16
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = ld_shared_v4(c_tile + sw128(t, q));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            o[2 * e] = e4m3x2_to_f16x2((uint16_t)(w[e] & 0xFFFFu));
            o[2 * e + 1] = e4m3x2_to_f16x2((uint16_t)(w[e] >> 16));
          }
          tmem_st8(a_tile + 8u * q, o);  // codes 16 q .. 16 q + 15 = TMEM columns 8 q .. 8 q + 7
        }
      }
      if (st.pass == 0) {
        tmem_wait_st();
        ++d2;
      }
      tc_fence_before();
      fence_async_shared();  // the in-place U split, for the MMA
      named_sync(1, 128);
      if (t == 0) mbar_arrive(&full[s]);
    }
  } else if (warp == 12) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t step = 0, e2 = 0, d2 = 0;
      for (Steps<DecParams> st(p, beg, end, q, S); st.valid() && !failed; st.next(), ++step) {
        const int s = step % kDStages;
        // D3 of p_{k-1} needs its P o c, which the epilogue forms at the block's start
        if (st.pass == 1 && st.i2 == 0 && !mbar_wait(pc_full, (st.k - 1) & 1u, kWaitLimit)) { failed = 1; break; }
        if (!mbar_wait(&full[s], (step / kDStages) & 1u, kWaitLimit)) { failed = 1; break; }
        const uint32_t u_tile = sbase + s * kDStageBytes + kDCodes;
        if (st.pass == 0) {
          // D2: T_c[128 x 64] = q_c . [U_hi | U_lo 2^11]   (f16)
          const int b = d2 & 1;
          if (d2 >= 2 && !mbar_wait(&t_empty[b], ((d2 >> 1) - 1) & 1u, kWaitLimit)) { failed = 1; break; }
          tc_fence_after();
          const uint32_t a_tile = tbase + kColA + 64u * (uint32_t)b;  // the converters' A tile d2 & 1
          const uint32_t d = tbase + (b ? kColT1 : kColT0);
#pragma unroll
          for (int kc = 0; kc < 8; ++kc) {  // K = 16 kc .. 16 kc + 15: A columns 8 kc .., U rows 16 kc ..
            const uint64_t bd = umma_desc_sw128(u_tile + kc * 16 * 128, 16, 1024);
            umma_f16_tmem_a(d, a_tile + 8u * kc, bd, kIdescD2, kc ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          umma_commit(&afree[b]);
          umma_commit(&t_full[b]);
          ++d2;
        } else {
          // D3: W[128 x 128] = Pc . U^T (three split products, bf16)
          const int b = (int)(e2 % kWBufs);
          if (e2 >= kWBufs && !mbar_wait(&w_empty[b], ((e2 / kWBufs) - 1) & 1u, kWaitLimit)) { failed = 1; break; }
          tc_fence_after();
          const uint32_t d = tbase + w_col(b);
          const int ak[6] = {0, 16, 32, 48, 0, 16};
          const int bk[6] = {0, 16, 0, 16, 32, 48};
#pragma unroll
          for (int q = 0; q < 6; ++q) {
            const uint64_t ad = umma_desc_sw128(pc_tile + ak[q] * 2, 16, 1024);
            const uint64_t bd = umma_desc_sw128(u_tile + bk[q] * 2, 16, 1024);
            umma_bf16(d, ad, bd, kIdescE2, q ? 1u : 0u);
          }
          umma_commit(&w_full[b]);
          ++e2;
        }
      }
    }
  } else {
    // ---------------- epilogue: warps 0-7 ----------------
    // Thread (r, h): row r = 32 (warp % 4) + lane (its TMEM lane); in D2 the
    // coefficients k = 16 h .. 16 h + 15, in D3 the columns 64 h .. 64 h + 63
    // of every 128-column chunk (h = warp / 4).  P of the panel in its first
    // pass stays in registers until the block that starts its second pass;
    // D3 writes its bf16 tile into an output tile for the store warp.
    const int h = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    __shared__ float coefs[2][33];  // by panel parity: see dec_coefs
    if (warp == 0 && beg < end) dec_coefs(p, beg, coefs[0], lane);  // p_0 (read after barriers)
    uint32_t step = 0, e2 = 0, d2 = 0, nx = 0;
    float P[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) P[k] = 0.0f;
    float a = 0.0f;
    bool stop = false;
    // E4M3: the chunk's fp32 block scale of this thread's row; NVFP4: the
    // tensor scale (the block scales are inside the widened values).  Loaded
    // one step ahead, so its memory latency overlaps the step before.
    auto scale_of = [&](const Steps<DecParams>& t) -> float {
      const DecJob& Jt = p.jobs[t.job()];
      const int64_t rw = (int64_t)t.panel() * kPanel + r;
      if (rw >= Jt.d_out) return 0.0f;
      return FMT == kFmtE4M3 ? __ldg(Jt.scales + rw * (Jt.d_in / kChunk) + t.chunk()) : __ldg(Jt.tscale);
    };
    Steps<DecParams> ahead(p, beg, end, q, S);
    float sc_next = ahead.valid() ? scale_of(ahead) : 0.0f;
    for (Steps<DecParams> st(p, beg, end, q, S); st.valid() && !stop; st.next(), ++step) {
      const int s = step % kDStages;
      const DecJob& J = p.jobs[st.job()];
      const int c = st.chunk();
      const int64_t row = (int64_t)st.panel() * kPanel + r;
      const bool live = row < J.d_out;
      const float sc = sc_next;
      ahead.next();
      sc_next = ahead.valid() ? scale_of(ahead) : 0.0f;
      if (st.block_start() && st.k >= 1) {
        // P of p_{k-1} is complete (in a cluster: this CTA's chunks of it,
        // summed over the cluster here): P o c -> bf16 hi/lo A operand of D3
        // (this half's 16 of the 32 columns of each part)
        if (CLUSTER) {
          stop = named_sync_or(2, 256, !cluster_sum16(P, xbuf, xfull, xempty, nx, S, q, r, h));
          if (stop) {
            failed = 1;
            break;
          }
        }
        // coefficients of p_{k-1} from its slot (formed a block ago)
        const float* cs = coefs[(st.k - 1) & 1];
        a = cs[32];
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float c0 = cs[16 * h + 2 * k], c1 = cs[16 * h + 2 * k + 1];
          float h0, l0, h1, l1;
          split_bf16(P[2 * k] * c0, h0, l0);
          split_bf16(P[2 * k + 1] * c1, h1, l1);
          hi[k] = pack_bf16x2(h0, h1);
          lo[k] = pack_bf16x2(l0, l1);
        }
        st_shared_v4(pc_tile + sw128(r, 2 * h), hi[0], hi[1], hi[2], hi[3]);
        st_shared_v4(pc_tile + sw128(r, 2 * h + 1), hi[4], hi[5], hi[6], hi[7]);
        st_shared_v4(pc_tile + sw128(r, 4 + 2 * h), lo[0], lo[1], lo[2], lo[3]);
        st_shared_v4(pc_tile + sw128(r, 5 + 2 * h), lo[4], lo[5], lo[6], lo[7]);
        fence_async_shared();
        mbar_arrive(pc_full);
        // the next panel's coefficients (its slot was last read a block ago)
        if (warp == 0 && beg + st.k < end) dec_coefs(p, beg + st.k, coefs[st.k & 1], lane);
      }
      if (st.pass == 0) {
        // D2 epilogue: P += s_c (T_hi + 2^-11 T_lo) for this half's 16 coefficients
        if (st.lidx() == 0) {
#pragma unroll
          for (int k = 0; k < 16; ++k) P[k] = 0.0f;
        }
        const int b = d2 & 1;
        stop = named_sync_or(2, 256, !mbar_wait(&t_full[b], (d2 >> 1) & 1u, kWaitLimit));
        if (stop) {
          failed = 1;
          break;
        }
        tc_fence_after();
        uint32_t th[16], tl[16];
        const uint32_t tcol = tbase + lane_off + (b ? kColT1 : kColT0) + 16 * h;
        tmem_ld16(tcol, th);
        tmem_ld16(tcol + 32, tl);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&t_empty[b]);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          P[k] = fmaf(sc, fmaf(__uint_as_float(tl[k]), 1.0f / kF16LoScale, __uint_as_float(th[k])), P[k]);
        if (not_finite(sc)) nonfin = 1;
        ++d2;
      } else {
        // D3 epilogue: G_hat = a s q + acc, into output tile o once its previous use is stored.
        // The stage is released as soon as every thread holds its 64 codes.
        const int b = (int)(e2 % kWBufs), o = (int)(e2 % kDOut);
        bool ok = mbar_wait(&w_full[b], (e2 / kWBufs) & 1u, kWaitLimit) &&
                  mbar_wait(&cfull[s], (step / kDStages) & 1u, kWaitLimit);
        if (e2 >= kDOut) ok = ok && mbar_wait(&ofree[o], ((e2 / kDOut) - 1) & 1u, kWaitLimit);
        const uint32_t c_tile = sbase + s * kDStageBytes;
        uint4 cv[4];  // E4M3: codes 64 h + 16 i .. + 15 of this row (in bounds whatever the waits gave)
        if (FMT == kFmtE4M3) {
#pragma unroll
          for (int i = 0; i < 4; ++i) cv[i] = ld_shared_v4(c_tile + sw128(r, 4 * h + i));
        }
        stop = named_sync_or(2, 256, !ok);
        if (stop) {
          failed = 1;
          break;
        }
        if (threadIdx.x == 0) mbar_arrive(&empty[s]);
        tc_fence_after();
        const uint32_t wcol = tbase + lane_off + w_col(b) + 64 * h;
        const uint32_t o_tile = otile + o * kDOutBytes;  // two [128][64] bf16 boxes, 128-byte swizzle
        const float as = a * sc;
        if (not_finite(sc)) nonfin = 1;
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
          uint32_t acc[32];
          tmem_ld32(wcol + g2 * 32, acc);
          tmem_wait_ld();
          // codes 64 h + 32 g2 .. + 31 of this row: two 16-byte chunks
          uint32_t o[16];
          if (FMT == kFmtE4M3) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint4 v = cv[2 * g2 + hh];
              const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f0 = e4m3x2_to_f32x2((uint16_t)(w[e] & 0xFFFFu));
                const float2 f1 = e4m3x2_to_f32x2((uint16_t)(w[e] >> 16));
                const int k = hh * 16 + e * 4;
                o[hh * 8 + 2 * e] = pack_bf16x2(fmaf(as, f0.x, __uint_as_float(acc[k])),
                                                fmaf(as, f0.y, __uint_as_float(acc[k + 1])));
                o[hh * 8 + 2 * e + 1] = pack_bf16x2(fmaf(as, f1.x, __uint_as_float(acc[k + 2])),
                                                    fmaf(as, f1.y, __uint_as_float(acc[k + 3])));
              }
            }
          } else {
            // NVFP4: columns 64 h + 32 g2 .. + 31 are blocks 4 h + 2 g2 and the next
            uint4 cq = make_uint4(0u, 0u, 0u, 0u);
            uint32_t sq = 0;
            if (live) {
              cq = __ldg(reinterpret_cast<const uint4*>(J.codes + row * (J.d_in / 2) + c * 64 + 32 * h + 16 * g2));
              sq = __ldg(reinterpret_cast<const uint16_t*>(J.sb + row * (J.d_in / 16) + c * 8 + 4 * h + 2 * g2));
            }
            float qv[32];
            nvfp4_block16_values(make_uint2(cq.x, cq.y), (uint8_t)(sq & 0xFFu), qv);
            nvfp4_block16_values(make_uint2(cq.z, cq.w), (uint8_t)(sq >> 8), qv + 16);
#pragma unroll
            for (int k = 0; k < 16; ++k)
              o[k] = pack_bf16x2(fmaf(as, qv[2 * k], __uint_as_float(acc[2 * k])),
                                 fmaf(as, qv[2 * k + 1], __uint_as_float(acc[2 * k + 1])));
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(o_tile + h * kGHalf + sw128(r, 4 * g2 + q), o[4 * q], o[4 * q + 1], o[4 * q + 2],
                         o[4 * q + 3]);
        }
        tc_fence_before();
        mbar_arrive(&w_empty[b]);
        fence_async_shared();
        mbar_arrive(&oready[o]);
        ++e2;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CLUSTER) cluster_sync_all();
  if (warp == 12) tmem_dealloc(tbase, kTmemCols);
  if (threadIdx.x == 0 && err && (failed || nonfin))
    atomicOr(err, (failed ? GIFT_DEV_TIMEOUT : 0u) | (nonfin ? GIFT_DEV_NONFINITE : 0u));
}

unsigned long long g_dec_attr[3][2] = {};
unsigned long long g_enc_attr[3][2] = {};

// One launch of `grid` clusters of S CTAs (S = 1: a plain launch).
template <class Prm>
cudaError_t launch_clusters(void (*kern)(Prm, uint32_t*), int smem, unsigned long long* attr, int grid, int S,
                            const Prm& P, uint32_t* err, cudaStream_t s) {
  cudaError_t e = ensure_smem_attr(kern, smem, attr);
  if (e != cudaSuccess) return e;
  if (S == 1) {
    kern<<<grid, kThreads, smem, s>>>(P, err);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(grid * S));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)S;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P, err);
}

// Clusters of S CTAs of this kernel that can be resident at once (0 if none).
template <class Prm>
int cluster_slots(void (*kern)(Prm, uint32_t*), int smem, unsigned long long* attr, int S, int* cache) {
  int& c = cache[S >> 2];  // S = 2 -> [0], S = 4 -> [1]
  if (c >= 0) return c;
  if (ensure_smem_attr(kern, smem, attr) != cudaSuccess) return c = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(S * kNumSMs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)S;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return c = std::min(n, kNumSMs);
}

int g_enc_slots[3][2] = {{-1, -1}, {-1, -1}, {-1, -1}};
int g_dec_slots[3][2] = {{-1, -1}, {-1, -1}, {-1, -1}};

int enc_slots(int fmt, int S) {
  if (S == 1) return kNumSMs;
  constexpr int m = enc_smem(true);
  switch (fmt) {
    case kFmtE4M3: return cluster_slots(whiten_encode_tc_kernel<kFmtE4M3, true>, m, &g_enc_attr[0][1], S, g_enc_slots[0]);
    case kFmtNvfp4Amax:
      return cluster_slots(whiten_encode_tc_kernel<kFmtNvfp4Amax, true>, m, &g_enc_attr[1][1], S, g_enc_slots[1]);
    case kFmtNvfp4: return cluster_slots(whiten_encode_tc_kernel<kFmtNvfp4, true>, m, &g_enc_attr[2][1], S, g_enc_slots[2]);
    default: return 0;
  }
}

int dec_slots(int fmt, int S) {
  if (S == 1) return kNumSMs;
  constexpr int m = dec_smem(true);
  switch (fmt) {
    case kFmtE4M3: return cluster_slots(whiten_decode_tc_kernel<kFmtE4M3, true>, m, &g_dec_attr[0][1], S, g_dec_slots[0]);
    case kFmtNvfp4: return cluster_slots(whiten_decode_tc_kernel<kFmtNvfp4, true>, m, &g_dec_attr[2][1], S, g_dec_slots[2]);
    default: return 0;
  }
}

template <int FMT>
cudaError_t enc_launch_fmt(int grid, const EncParams& P, uint32_t* err, cudaStream_t s) {
  const int f = FMT == kFmtE4M3 ? 0 : FMT == kFmtNvfp4Amax ? 1 : 2;
  if (P.split > 1)
    return launch_clusters(whiten_encode_tc_kernel<FMT, true>, enc_smem(true), &g_enc_attr[f][1], grid, P.split, P,
                           err, s);
  return launch_clusters(whiten_encode_tc_kernel<FMT, false>, enc_smem(false), &g_enc_attr[f][0], grid, 1, P, err, s);
}

template <int FMT>
cudaError_t dec_launch_fmt(int grid, const DecParams& P, uint32_t* err, cudaStream_t s) {
  const int f = FMT == kFmtE4M3 ? 0 : 2;
  if (P.split > 1)
    return launch_clusters(whiten_decode_tc_kernel<FMT, true>, dec_smem(true), &g_dec_attr[f][1], grid, P.split, P,
                           err, s);
  return launch_clusters(whiten_decode_tc_kernel<FMT, false>, dec_smem(false), &g_dec_attr[f][0], grid, 1, P, err, s);
}

// One launch runs layers of one format (its kernel instantiation).
cudaError_t enc_launch(int fmt, int grid, const EncParams& P, uint32_t* err, cudaStream_t s) {
  switch (fmt) {
    case kFmtE4M3: return enc_launch_fmt<kFmtE4M3>(grid, P, err, s);
    case kFmtNvfp4Amax: return enc_launch_fmt<kFmtNvfp4Amax>(grid, P, err, s);
    case kFmtNvfp4: return enc_launch_fmt<kFmtNvfp4>(grid, P, err, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t dec_launch(int fmt, int grid, const DecParams& P, uint32_t* err, cudaStream_t s) {
  switch (fmt) {
    case kFmtE4M3: return dec_launch_fmt<kFmtE4M3>(grid, P, err, s);
    case kFmtNvfp4: return dec_launch_fmt<kFmtNvfp4>(grid, P, err, s);
    default: return cudaErrorInvalidValue;
  }
}

// Longest-processing-time-first assignment of panels to `slots` clusters of S
// CTAs (S = 1: single CTAs).  A panel costs each CTA of its cluster at most
// ceil(nc / S) steps per pass.  Returns the clusters used (or -1) and the
// largest per-cluster cost in *makespan; off / ids are written only if given.
int schedule(const TcLayer* layers, int n, uint16_t* off, uint16_t* ids, int max_ids, int slots, int S,
             long* makespan) {
  static thread_local std::vector<std::pair<int, uint16_t>> items;  // (cost, id), reused across calls
  static thread_local std::vector<int> owner;
  items.clear();
  for (int l = 0; l < n; ++l) {
    const int np = (layers[l].d_out + kPanel - 1) / kPanel;
    const int nc = layers[l].d_in / kChunk;
    for (int q = 0; q < np; ++q) items.push_back({(nc + S - 1) / S, (uint16_t)((l << 8) | q)});
  }
  if ((int)items.size() > max_ids || slots <= 0) return -1;
  std::stable_sort(items.begin(), items.end(),
                   [](const std::pair<int, uint16_t>& x, const std::pair<int, uint16_t>& y) { return x.first > y.first; });
  const int grid = std::min<int>(slots, (int)items.size());
  using E = std::pair<long, int>;
  std::priority_queue<E, std::vector<E>, std::greater<E>> heap;
  for (int b = 0; b < grid; ++b) heap.push({0, b});
  owner.resize(items.size());
  long worst = 0;
  for (size_t i = 0; i < items.size(); ++i) {
    E e = heap.top();
    heap.pop();
    owner[i] = e.second;
    worst = std::max(worst, e.first + items[i].first);
    heap.push({e.first + items[i].first, e.second});
  }
  if (makespan) *makespan = worst;
  if (off && ids) {
    // cluster b's panels, in the longest-first order they were assigned
    std::vector<int> cnt(grid + 1, 0);
    for (int o : owner) ++cnt[o + 1];
    for (int b = 0; b < grid; ++b) cnt[b + 1] += cnt[b];
    for (int b = 0; b <= grid; ++b) off[b] = (uint16_t)cnt[b];
    for (size_t i = 0; i < items.size(); ++i) ids[cnt[owner[i]]++] = items[i].second;
  }
  return grid;
}

// Cluster size for a launch.  A CTA that owns a panel runs 2 nc chunk steps
// (both passes); with a cluster of S CTAs per panel it runs 2 ceil(nc / S),
// plus a fixed cost of the cluster launch and the partial-P exchange that
// measured, on B200, about as long as kSplitCost[S] chunk steps.  A split is
// taken only when every cluster gets at most one panel (a second panel would
// repeat the exchange and the pipeline refill) and it is at least a tenth
// faster by that estimate; a launch of many panels keeps single CTAs.
constexpr int kSplitCost2 = 6, kSplitCost4 = 15;

template <class SlotFn>
int plan(const TcLayer* layers, int n, uint16_t* off, uint16_t* ids, int max_ids, SlotFn slots_for, int* split) {
  int min_nc = 1 << 30, max_nc = 0, panels = 0;
  for (int l = 0; l < n; ++l) {
    min_nc = std::min(min_nc, layers[l].d_in / kChunk);
    max_nc = std::max(max_nc, layers[l].d_in / kChunk);
    panels += (layers[l].d_out + kPanel - 1) / kPanel;
  }
  int best_s = 1;
  if (panels < kNumSMs) {
    const long est1 = 2L * max_nc;
    long best = est1;
    for (int S : {2, 4}) {
      if (S > min_nc) break;
      const int slots = slots_for(S);
      if (slots <= 0 || panels > slots) continue;
      const long est = 2L * ((max_nc + S - 1) / S) + (S == 2 ? kSplitCost2 : kSplitCost4);
      if (10 * est < 9 * est1 && est < best) {
        best = est;
        best_s = S;
      }
    }
  }
  *split = best_s;
  return schedule(layers, n, off, ids, max_ids, best_s == 1 ? kNumSMs : slots_for(best_s), best_s, nullptr);
}

}  // namespace

bool tc_codec_available() { return tmap_encoder() != nullptr; }

namespace {
// One thread per U row: the same parts the converter warps form in shared
// memory (store_u_split_bf16 / store_u_split_f16), written to global memory.
__global__ void __launch_bounds__(128) split_u_kernel(const float* __restrict__ U, int64_t d_in,
                                                      uint16_t* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= d_in) return;
  const float4* src = reinterpret_cast<const float4*>(U + i * 32);
  float u[32];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 v = __ldg(src + q);
    u[4 * q] = v.x;
    u[4 * q + 1] = v.y;
    u[4 * q + 2] = v.z;
    u[4 * q + 3] = v.w;
  }
  uint32_t bh[16], bl[16], fh[16], fl[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float h0, l0, h1, l1;
    split_bf16(u[2 * k], h0, l0);
    split_bf16(u[2 * k + 1], h1, l1);
    bh[k] = pack_bf16x2(h0, h1);
    bl[k] = pack_bf16x2(l0, l1);
    const float g0 = __half2float(__float2half_rn(u[2 * k]));
    const float g1 = __half2float(__float2half_rn(u[2 * k + 1]));
    fh[k] = pack_f16x2(g0, g1);
    fl[k] = pack_f16x2((u[2 * k] - g0) * kF16LoScale, (u[2 * k + 1] - g1) * kF16LoScale);
  }
  uint4* b = reinterpret_cast<uint4*>(out + i * 64);
  uint4* f = reinterpret_cast<uint4*>(out + (d_in + i) * 64);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    b[q] = make_uint4(bh[4 * q], bh[4 * q + 1], bh[4 * q + 2], bh[4 * q + 3]);
    b[4 + q] = make_uint4(bl[4 * q], bl[4 * q + 1], bl[4 * q + 2], bl[4 * q + 3]);
    f[q] = make_uint4(fh[4 * q], fh[4 * q + 1], fh[4 * q + 2], fh[4 * q + 3]);
    f[4 + q] = make_uint4(fl[4 * q], fl[4 * q + 1], fl[4 * q + 2], fl[4 * q + 3]);
  }
}
}  // namespace

cudaError_t launch_split_u(const float* U, int64_t d_in, uint16_t* U_split, cudaStream_t s) {
  if (d_in <= 0) return cudaSuccess;
  split_u_kernel<<<(unsigned)((d_in + 127) / 128), 128, 0, s>>>(U, d_in, U_split);
  return cudaGetLastError();
}

// Layers [0, cnt) of one launch: the same format, at most kMaxJobs layers and
// kMaxPanels panels, each layer at most 256 panels (0: the first layer is
// larger and is coded in parts of 256 panels).
// Tensor map of a layer's U tiles: fp32 [d_in][32] (split in the kernel), or
// the pre-split [2 d_in][64] 16-bit rows; both give 128-byte rows in 128-row boxes.
static bool make_u_tmap(CUtensorMap* m, const TcLayer& L) {
  if (L.U_split)
    return make_tmap_2d(m, L.U_split, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, 2 * (uint64_t)L.d_in, 64, kChunk, 64);
  return make_tmap_2d(m, L.U, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)L.d_in, 32, kChunk, 32);
}

static int group_count(const TcLayer* layers, int n) {
  int cnt = 0, panels = 0;
  while (cnt < n && cnt < kMaxJobs && layers[cnt].fmt == layers[0].fmt &&
         (layers[cnt].U_split != nullptr) == (layers[0].U_split != nullptr)) {
    const int np = (layers[cnt].d_out + kPanel - 1) / kPanel;
    if (np > 256 || panels + np > kMaxPanels) break;
    panels += np;
    ++cnt;
  }
  return cnt;
}

int tc_codec_split(const TcLayer* layers, int n, bool encode) {
  if (n <= 0) return -1;
  TcLayer part = layers[0];
  const TcLayer* g = layers;
  int cnt = group_count(layers, n);
  if (cnt == 0) {
    part.d_out = std::min(part.d_out, 256 * kPanel);
    g = &part;
    cnt = 1;
  }
  static thread_local uint16_t off[kNumSMs + 1], ids[kMaxPanels];
  const int fmt = g[0].fmt;
  int S = 1;
  const int grid = encode ? plan(g, cnt, off, ids, kMaxPanels, [fmt](int k) { return enc_slots(fmt, k); }, &S)
                          : plan(g, cnt, off, ids, kMaxPanels, [fmt](int k) { return dec_slots(fmt, k); }, &S);
  return grid <= 0 ? -1 : S;
}

cudaError_t launch_whiten_encode_tc(const TcLayer* layers, int n, uint32_t* err, cudaStream_t s,
                                    uint32_t stall_polls) {
  cudaError_t e = cudaSuccess;
  for (int base = 0; base < n;) {
    // pack as many layers as fit one launch
    const int cnt = group_count(layers + base, n - base);
    if (cnt == 0) {
      // a single layer with more than 256 panels: split it by rows
      const TcLayer& L = layers[base];
      const int rows = 256 * kPanel;
      for (int r0 = 0; r0 < L.d_out; r0 += rows) {
        TcLayer part = L;
        part.d_out = std::min(rows, L.d_out - r0);
        part.G = (const __nv_bfloat16*)L.G + (int64_t)r0 * L.d_in;
        if (L.fmt == kFmtE4M3) {
          part.codes = L.codes + (int64_t)r0 * L.d_in;
          part.scales = L.scales + (int64_t)r0 * (L.d_in / kChunk);
        } else {
          part.codes = L.codes + (int64_t)r0 * (L.d_in / 2);
          part.block_scales = L.block_scales + (int64_t)r0 * (L.d_in / 16);
        }
        if ((e = launch_whiten_encode_tc(&part, 1, err, s, stall_polls)) != cudaSuccess) return e;
      }
      ++base;
      continue;
    }
    static thread_local EncParams P;
    for (int l = 0; l < cnt; ++l) {
      const TcLayer& L = layers[base + l];
      EncJob& J = P.jobs[l];
      if (!make_tmap_2d(&J.tmG, L.G, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)L.d_out, (uint64_t)L.d_in,
                        kPanel, 64) ||
          !make_u_tmap(&J.tmU, L) ||
          (L.fmt == kFmtE4M3 && !make_tmap_2d(&J.tmC, L.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.d_out,
                                              (uint64_t)L.d_in, kPanel, kChunk)))
        return cudaErrorInvalidValue;
      J.U = L.U;
      J.lambda = L.lambda;
      J.rho = L.rho;
      J.codes = L.codes;
      J.sb = L.block_scales;
      J.tscale = L.tensor_scale;
      J.fmt = L.fmt;
      J.scales = L.scales;
      J.d_out = L.d_out;
      J.d_in = L.d_in;
      J.rank = L.rank;
    }
    const int fmt = layers[base].fmt;
    const int grid = plan(layers + base, cnt, P.sched_off, P.sched_ids, kMaxPanels,
                          [fmt](int S) { return enc_slots(fmt, S); }, &P.split);
    if (grid <= 0) return cudaErrorInvalidValue;
    P.stall_polls = stall_polls;
    P.presplit = layers[base].U_split != nullptr;
    if ((e = enc_launch(fmt, grid, P, err, s)) != cudaSuccess) return e;
    base += cnt;
  }
  return cudaSuccess;
}



cudaError_t launch_whiten_decode_tc(const TcLayer* layers, int n, uint32_t* err, cudaStream_t s,
                                    uint32_t stall_polls) {
  cudaError_t e = cudaSuccess;
  for (int base = 0; base < n;) {
    const int cnt = group_count(layers + base, n - base);
    if (cnt == 0) {
      const TcLayer& L = layers[base];
      const int rows = 256 * kPanel;
      for (int r0 = 0; r0 < L.d_out; r0 += rows) {
        TcLayer part = L;
        part.d_out = std::min(rows, L.d_out - r0);
        part.G_hat = (__nv_bfloat16*)L.G_hat + (int64_t)r0 * L.d_in;
        if (L.fmt == kFmtE4M3) {
          part.codes = L.codes + (int64_t)r0 * L.d_in;
          part.scales = L.scales + (int64_t)r0 * (L.d_in / kChunk);
        } else {
          part.codes = L.codes + (int64_t)r0 * (L.d_in / 2);
          part.block_scales = L.block_scales + (int64_t)r0 * (L.d_in / 16);
        }
        if ((e = launch_whiten_decode_tc(&part, 1, err, s, stall_polls)) != cudaSuccess) return e;
      }
      ++base;
      continue;
    }
    static thread_local DecParams P;
    for (int l = 0; l < cnt; ++l) {
      const TcLayer& L = layers[base + l];
      DecJob& J = P.jobs[l];
      if ((L.fmt == kFmtE4M3 && !make_tmap_2d(&J.tmC, L.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)L.d_out,
                                              (uint64_t)L.d_in, kPanel, kChunk)) ||
          !make_u_tmap(&J.tmU, L) ||
          !make_tmap_2d(&J.tmO, L.G_hat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)L.d_out, (uint64_t)L.d_in,
                        kPanel, 64))
        return cudaErrorInvalidValue;
      J.U = L.U;
      J.lambda = L.lambda;
      J.rho = L.rho;
      J.scales = L.scales;
      J.codes = L.codes;
      J.sb = L.block_scales;
      J.tscale = L.tensor_scale;
      J.fmt = L.fmt;
      J.d_out = L.d_out;
      J.d_in = L.d_in;
      J.rank = L.rank;
    }
    const int fmt = layers[base].fmt;
    const int grid = plan(layers + base, cnt, P.sched_off, P.sched_ids, kMaxPanels,
                          [fmt](int S) { return dec_slots(fmt, S); }, &P.split);
    if (grid <= 0) return cudaErrorInvalidValue;
    P.stall_polls = stall_polls;
    P.presplit = layers[base].U_split != nullptr;
    if ((e = dec_launch(fmt, grid, P, err, s)) != cudaSuccess) return e;
    base += cnt;
  }
  return cudaSuccess;
}

}  // namespace gift
