// gemm_sm100.cu -- device-scheduled grouped GEMM on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA), bf16 operands, fp32 accumulation, with the
// SwiGLU forward and backward fused into the epilogues; and the bf16 expert
// FFN forward/backward built from it.
//
// Page: "Ai2 Olmo-core 3：MoE训练吞吐量提升2.7倍的秘诀" (kongchang.com), section
// 路由不只是模型问题，更是系统问题: a device-scheduled grouped GEMM handles the
// uneven per-expert shapes produced by routing, packing the small GEMMs of all
// experts into one kernel without padding; group sizes never go back to the host.
//
// Kernel structure (one CTA per SM, persistent; 10 warps):
//   warp 0      TMA producer (one thread): A/B tiles -> S-stage smem ring
//   warp 1      MMA issuer (one thread issues tcgen05.mma M=128 N=BN K=16;
//               the warp zeroes ragged K tails of weight-gradient tiles)
//   warps 2..9  epilogue, two warps per TMEM lane quarter, each on half of the
//               columns: tcgen05.ld TMEM -> registers -> fused math -> global
// TMEM holds two BN-column fp32 accumulators so the epilogue of one tile
// overlaps the main loop of the next.
//
// Tile scheduler: each CTA reads offsets[0..E] from device memory into shared
// memory and builds the per-expert tile prefix itself; tile t of the launch is
// then found by a binary search.  The host never learns the group sizes: it
// launches one CTA per SM and idle CTAs exit.
//   GROUP_M (forward, dgrad): expert g owns rows [off[g], off[g+1]) of A and
//     of the output; M tiles of 128 rows; rows of a tile beyond the segment
//     are computed but not stored.
//   GROUP_K (wgrad): expert g owns the K range [off[g], off[g+1]) of both
//     operands (the token axis); the rows of the last K block that belong to
//     the next expert are zeroed in shared memory before the MMA reads them;
//     an expert without rows writes a zero tile.
//
// Shared-memory operand layouts (128-byte swizzle, matching the TMA swizzle):
//   K-major  (rows of K contiguous): 128-B rows, 8-row groups 1024 B apart
//            (SBO = 1024); the K=16 slices of a 64-wide stage start 32 B apart.
//   MN-major (rows of M/N contiguous, K along rows): boxes of 64 M/N elements
//            x 64 K rows; 8-K-row groups 1024 B apart (SBO), 64-element M/N
//            blocks 8192 B apart (LBO); K=16 slices start 2048 B apart.
//
// Every mbarrier wait is bounded (common.cuh); on a timeout the kernel records
// MOE_ERR_TIMEOUT, raises a CTA-wide abort flag, waits (bounded) for its own
// TMA loads and MMAs in flight, frees TMEM and returns.
#include "common.cuh"
#include "mx_common.cuh"
#include "internal.h"

#include <cudaTypedefs.h>
#include <stdlib.h>

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr uint32_t kABytes = BM * BK * 2;  // 16 KB

enum : int {
  EPI_SWIGLU_FWD = 0,  // gate|up accumulators -> a, u, h = silu(a) u
  EPI_STORE = 1,       // bf16 store
  EPI_SWIGLU_BWD = 2,  // dh -> da, du (loads a, u)
  EPI_WGRAD = 3,       // per-group weight gradient, fp32 (TMA store) or bf16
  EPI_ROUTER = 4,      // logits -> softmax, top-k, block counts and ranks
  EPI_ROUTER_DX = 5    // dx = acc + sum_j dx_perm[slot_row[t, j]]
};

constexpr int kRouterKMax = 8;  // top-k kept in registers by the router epilogue


struct GemmParams {
  CUtensorMap tmA;
  CUtensorMap tmB;
  CUtensorMap tmOut;       // output: bf16 boxes of 64 columns x 16 rows, or fp32 (wgrad) 32 x 16
  const int32_t* offsets;
  int E;
  int M;        // GROUP_K: output rows per expert
  int N;        // GROUP_M: output columns (SwiGLU forward: f); GROUP_K: output columns
  int K;        // GROUP_M: reduction length
  int b_rows;   // GROUP_M: rows of B per expert in the flattened weight tensor
  int f;        // d_ff
  __nv_bfloat16* out;
  int64_t ld_out;
  float* out_f32;          // EPI_WGRAD with fp32 output (else out)
  const __nv_bfloat16* act;
  int64_t ld_act;
  int64_t out_group;       // EPI_WGRAD: elements per expert
  int accumulate;          // EPI_WGRAD: add into the output instead of overwriting it
  int* status;
  // EPI_ROUTER (one group of rows_total tokens; N = number of experts)
  int rows_total;
  int topk;
  int nb;                  // 128-token blocks
  const float* bias;
  float* logits;
  int32_t* topk_idx;
  float* topk_gate;
  int32_t* blockcounts;    // [N][nb]
  int32_t* localrank;      // [rows_total][topk]
  // GROUP_K without offsets: groups are consecutive splits of `split` rows
  int split;
  // GROUP_K with offsets: a group of c > kchunk rows is cut into ns K ranges of ck rows
  // (wgrad_split); tile (g, range j) then writes an fp32 partial sum to slot
  // (slot prefix of g) + j of `part` ([slots * M, N], tensor map tmPart), and
  // wgrad_reduce adds the ranges in order.  kchunk = 0: no cut.
  int kchunk;
  float* part;
  CUtensorMap tmPart;
  // MXFP8 CTA pairs: the scale atoms as [2 x atoms, 256] byte tensors (box 256 x 2 = one
  // atom), so that they load with the pair's TMA form onto the leader's barrier
  CUtensorMap tmSfa, tmSfb;
  // Failure-path test hooks (0 = off): the limit of every bounded wait, and a ring
  // iteration at which CTA 0's producer skips its loads and its arrival, so that the MMA
  // warp's wait runs out (see gemm_test_hooks).
  uint64_t wait_ns;
  int drop_it;
  // EPI_ROUTER_DX
  const int32_t* slot_row; // [rows_total][topk]
  // MXFP8 operand copies written by the epilogue (mx_q_r non-null): the row copy
  // [rows][K] with row-tile atoms, and the token-block copy [K][mx_rp] (column-major,
  // stage-padded) with stage atoms.  EPI_SWIGLU_BWD: [da | du] (K = 2f) instead of bf16
  // (`out`, when also set, receives the bf16 rows as well: a diagnostic form);
  // EPI_SWIGLU_FWD: h (K = f), besides a | u | h in bf16
  uint8_t* mx_q_r;
  uint8_t* mx_s_r;
  uint8_t* mx_q_c;
  uint8_t* mx_s_c;
  int64_t mx_rp;
  // MXFP8 operands: E8M0 scales as 512-byte MMA atoms (128 rows x 4 blocks of 32
  // along K), in the order the producer reads them (see the MXFP8 producer).
  const uint8_t* sfa;
  const uint8_t* sfb;
};

template <int BN, bool PAIR = false, int EPI = 1, bool FP8 = false> struct Cfg {
  // PAIR: a CTA pair computes a 256-row tile; each CTA holds its 128 A rows and half
  // of the BN B rows (cta_group::2).
  // FP8 (MXFP8): 128 E4M3 elements (128 bytes) of K per stage, plus the stage's scale
  // atoms for A (512 B) and B (BN / 128 x 512 B); each stage's scales go to one of 16
  // slots of 8 TMEM columns after the accumulators.
  static constexpr int kBKe = FP8 ? 128 : BK;  // K elements per stage
  static constexpr uint32_t kBBytes = (PAIR ? BN / 2 : BN) * 128;
  // FP8: A atom (512 B) + the B atoms (BN/128 of them; in a CTA pair each CTA holds the
  // scales of all BN columns, as the pair's block-scaled MMA reads them from each CTA's
  // TMEM), padded to keep stages 1024-byte aligned
  static constexpr uint32_t kSfB = (BN / 128) * 512;
  static constexpr uint32_t kSfLoad = FP8 ? 512 + kSfB : 0;   // bytes loaded per stage
  static constexpr uint32_t kSfBytes = FP8 ? ((kSfLoad + 1023) / 1024) * 1024 : 0;
  static constexpr uint32_t kStage = kABytes + kBBytes + kSfBytes;
  static_assert(kStage % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  // accumulator buffers: two (the epilogue of one tile overlaps the main loop of the
  // next), except for 256-wide MXFP8 tiles, whose scale columns leave room for one
  static constexpr int kAccBufs = (FP8 && BN == 256) ? 1 : 2;
  // FP8: 4 slots of 16 scale columns after the accumulators (A at +0, B atoms at +4, +8),
  // used in rotation.  The tensor pipe runs one thread's scale copies and MMAs in issue
  // order, so a slot is rewritten only after the MMAs of the stage that used it.
  static constexpr uint32_t kSfCol = kAccBufs * BN;
  static constexpr uint32_t kSfSlots = 4;
  static_assert(!FP8 || kSfCol + kSfSlots * 16 <= 512, "scale slots fit in TMEM");
  // columns after the scale slots, free for the epilogue (a single 256-wide accumulator
  // leaves 192: three 32-column chunks for each of the two warps of a lane quarter)
  static constexpr uint32_t kSpareCol = kSfCol + kSfSlots * 16;
  static constexpr uint32_t kTmemCols = FP8 ? 512 : 2 * BN;
  static constexpr int kBoxRows = BN < 128 ? BN : 128;  // rows of one K-major B box
  static constexpr int kTileM = PAIR ? 2 * BM : BM;     // rows of one scheduled tile
  // TMA-store staging per epilogue warp: bf16 outputs use two 2 KB slots, the fp32
  // weight gradient one; the router epilogues store directly.
  // (MXFP8 weight gradients, whose short K makes the fp32 stores the longer part of a
  // tile, keep two slots per warp as well)
  static constexpr size_t kStoreBytes =
      EPI == EPI_WGRAD ? (FP8 ? 8 * 4096 : 8 * 2048)
                       : ((EPI == EPI_ROUTER || EPI == EPI_ROUTER_DX) ? 0 : 8 * 4096);
  // shared memory after the stage ring: barriers (256 B), offsets and tile prefix
  // (2 x 1025 ints), router histogram (128 x kRouterKMax ints), then the 1024-aligned
  // staging area; as many stages as fit (up to 6)
  // weight-gradient kernels keep a third per-group array (split slot prefix)
  static constexpr size_t kExtra = EPI == EPI_WGRAD ? 1025 * 4 : 0;
  static constexpr size_t kFixed = 1024 + 256 + 2 * 1025 * 4 + 128 * kRouterKMax * 4 + kExtra + 1024 + kStoreBytes;
  static constexpr int kStages = (232448 - kFixed) / kStage > 6 ? 6 : (int)((232448 - kFixed) / kStage);
  static constexpr size_t kOffMisc = (size_t)kStages * kStage;
  static constexpr size_t kOffSoff = kOffMisc + 256;
  static constexpr size_t kOffSel = kOffSoff + 2 * 1025 * 4;
  static constexpr size_t kOffExtra = kOffSel + 128 * kRouterKMax * 4;
  static constexpr size_t kOffStore = (kOffExtra + kExtra + 1023) & ~size_t(1023);
  static constexpr size_t kSmem = 1024 + kOffStore + kStoreBytes;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert(128 * kRouterKMax * 4 >= 4 * 256 * 4, "router histogram fits the selection area");
};

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// ---- MXFP8: block-scaled E4M3 MMA (K = 32 per instruction, one E8M0 scale per row per
// 32 K) and the shared-memory -> TMEM copy of a 128-row x 4-block scale atom.
__device__ __forceinline__ void umma_mxf8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accum, uint32_t tsfa, uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum), "r"(tsfa), "r"(tsfb));
}
// 32 rows x 16 bytes from shared memory, broadcast to the four 32-lane quarters.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc_src) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc_src)
               : "memory");
}
// descriptor of a 512-byte scale atom: 32 rows of 16 bytes, no swizzle (8-row groups 128 B apart)
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 16) |
         ((uint64_t)(128 >> 4) << 32) | (1ull << 46);
}

// ---- CTA-pair (cta_group::2) forms
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// TMA load into this CTA's shared memory, completing on the leader CTA's barrier.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* tm, int x, int y,
                                                 uint32_t leader_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(leader_bar)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                               uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void umma_mxf8_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                               uint32_t accum, uint32_t tsfa, uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum), "r"(tsfa), "r"(tsfb));
}
// each CTA of the pair copies the atom at this shared-memory offset into its own TMEM
__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc_src) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc_src)
               : "memory");
}
// Arrive on the barrier at this offset in both CTAs of the pair once the MMAs are done.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)), "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

#define MOE_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                  "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define MOE_T8(i) "+r"(r[i + 0]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), \
                  "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : MOE_R8(0), MOE_R8(8), MOE_R8(16), MOE_R8(24)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : MOE_R8(0), MOE_R8(8)
      : "r"(taddr));
}
#define MOE_S8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                  "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])
// 32 consecutive fp32 columns of this thread's TMEM lane, written from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      MOE_S8(0), MOE_S8(8), MOE_S8(16), MOE_S8(24)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_tie16(uint32_t (&r)[16]) {
  asm volatile("" : MOE_T8(0), MOE_T8(8));
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, int x, int y, const void* smem_src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(x), "r"(y), "r"(smem_u32(smem_src))
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The same box added element-wise into global memory (fp32 adds in L2, one per element)
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* tm, int x, int y,
                                                  const void* smem_src) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(tm)),
      "r"(x), "r"(y), "r"(smem_u32(smem_src))
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_read_le1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Orders every later use of r after the preceding wait::ld.
__device__ __forceinline__ void tmem_tie(uint32_t (&r)[32]) {
  asm volatile("" : MOE_T8(0), MOE_T8(8), MOE_T8(16), MOE_T8(24));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ void store_64B(void* dst, const uint32_t (&v)[16]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
// logistic function with the fast exponential and the fast division intrinsics (about two
// ulp in fp32, far below the bf16 rounding of every value it feeds)
__device__ __forceinline__ float sigmoidf_(float a) { return __fdividef(1.f, 1.f + __expf(-a)); }
// 32 bf16 of a (at col) and of u (at f + col) from one row of the saved activations, as
// 32-byte loads (one whole sector each: the buffer is 32-byte aligned, a check of the call,
// and col, f and the row pitch 3 f keep every piece so) that do not allocate in L1.  These
// loads run while the next tile's MMAs do; with 16-byte loads the MMAs of the
// SwiGLU-backward GEMM issued about 8 % slower.
__device__ __forceinline__ void ldg32_na(const __nv_bfloat16* p, uint32_t* r) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}
__device__ __forceinline__ void load_au(const __nv_bfloat16* arow, int col, int f,
                                        uint32_t (&av)[16], uint32_t (&uv)[16]) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    ldg32_na(arow + col + 16 * i, av + 8 * i);
    ldg32_na(arow + f + col + 16 * i, uv + 8 * i);
  }
}

// Store a 16-row x 64-column bf16 box whose rows are held by lanes 16*hh .. 16*hh+15
// (each lane: its row's 64 values as 32 packed bf16x2 words).  The box is staged in one
// of the warp's two 2 KB slots with the 128-byte swizzle and written by one TMA store
// (whole lines, asynchronous).  A box that reaches past the valid rows (the last tile
// of an expert: the next rows belong to the next expert) is written row by row instead.
__device__ __forceinline__ void put_box_bf16(uint8_t* wbuf, uint32_t& slot, const CUtensorMap* tm,
                                             const uint32_t (&v)[32], int hh, int x, int y,
                                             int valid_rows, __nv_bfloat16* row_dst) {
  const int lane = threadIdx.x & 31;
  if (valid_rows <= 0) return;
  const bool mine = (lane >> 4) == hh;
  const int r = lane & 15;
  if (valid_rows < 16) {
    if (mine && r < valid_rows) {
      uint4* d = reinterpret_cast<uint4*>(row_dst);
#pragma unroll
      for (int j = 0; j < 8; ++j) d[j] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
    return;
  }
  uint8_t* buf = wbuf + (slot & 1) * 2048;
  if (lane == 0) tma_store_wait_read_le1();  // the store that used this slot has read it
  __syncwarp();
  if (mine) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint4*>(buf + r * 128 + ((j ^ (r & 7)) * 16)) =
          make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) tma_store_2d(tm, x, y, buf);
  ++slot;
}

// MXFP8 copies of one 32 x 32 block of an activation that a warp holds: lane = row of a
// 32-token block (rows past the segment's end held as zero), pk = the row's 32 bf16 values
// of this block's columns.  Writes the row copy (32 codes + one scale per valid row) and
// the token-block copy (per column, the 32 codes down the block's rows as one 32-byte run
// of the column-major copy, + one scale), exactly as the activation quantiser does.  A
// block with no row in the segment (`live` false; its stage still exists) gets zero codes
// and 2^0 scales.  s_tr: 32 x 17 words of this warp's shared memory.
//   q_r_row:  row copy at this row and the block's first column (unused if !row_valid)
//   at_r:     this row's scale byte in its row-tile atom (unused if !row_valid)
//   q_c_blk:  token-block copy at the block's first column and first row
//   at_c:     the stage atom of the block's 128-column slab; c0: the block's first column
//             within that slab (0, 32, 64, 96); tb: the token block within the stage
// 32 bytes (one sector) in one store; p is 32-byte aligned
__device__ __forceinline__ void stg32(void* p, const uint32_t* r) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void mx_emit_block(const uint32_t* pk, bool row_valid, bool live,
                                              uint8_t* q_r_row, uint8_t* at_r, uint8_t* q_c_blk,
                                              int64_t rp, uint8_t* at_c, int c0, int tb,
                                              uint32_t* s_tr) {
  const int lane = threadIdx.x & 31;
  if (row_valid) {
    // the row: maximum on packed bf16 pairs (exact), then 32 codes and the scale
    __nv_bfloat162 am = __float2bfloat162_rn(0.f);
#pragma unroll
    for (int i = 0; i < 16; ++i) am = __hmax2(am, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&pk[i])));
    const int ex = block_exponent(fmaxf(__low2float(am), __high2float(am)));
    const float mul = pow2_neg(ex);
    uint32_t w8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w8[i] = e4m3_pair(bf_hi(pk[2 * i]) * mul, bf_lo(pk[2 * i]) * mul) |
              (e4m3_pair(bf_hi(pk[2 * i + 1]) * mul, bf_lo(pk[2 * i + 1]) * mul) << 16);
    stg32(q_r_row, w8);
    *at_r = (uint8_t)(ex + 127);
  }
  // columns: the block passes through shared memory (row `lane` at a pitch of 17 words), and
  // lane (cp, rh) takes the column pair 2 cp, 2 cp + 1 over rows 16 rh .. 16 rh + 15 (the
  // reads of one step hit 32 distinct banks); the pair's two lanes combine their maxima
  __syncwarp();
#pragma unroll
  for (int w = 0; w < 16; ++w) s_tr[lane * 17 + w] = row_valid ? pk[w] : 0u;
  __syncwarp();
  const int cp = lane >> 1, rh = lane & 1;
  uint32_t cw[16];
  __nv_bfloat162 cm = __float2bfloat162_rn(0.f);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    cw[i] = s_tr[(16 * rh + i) * 17 + cp];
    cm = __hmax2(cm, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&cw[i])));
  }
  const uint32_t cmu = *reinterpret_cast<uint32_t*>(&cm);
  const uint32_t oth = __shfl_xor_sync(0xffffffffu, cmu, 1);
  cm = __hmax2(cm, *reinterpret_cast<const __nv_bfloat162*>(&oth));
  const int ex0 = block_exponent(__low2float(cm)), ex1 = block_exponent(__high2float(cm));
  const float m0 = pow2_neg(ex0), m1 = pow2_neg(ex1);
  // codes of rows 16 rh + 4 j .. + 3: column 2 cp's bytes in o0, column 2 cp + 1's in o1
  uint32_t o0[4], o1[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w = cw[4 * j + i];
      pr[i] = e4m3_pair(bf_hi(w) * m1, bf_lo(w) * m0);
    }
    const uint32_t x = pr[0] | (pr[1] << 16), y = pr[2] | (pr[3] << 16);
    o0[j] = live ? __byte_perm(x, y, 0x6420) : 0u;
    o1[j] = live ? __byte_perm(x, y, 0x7531) : 0u;
  }
  // the pair swaps halves so that lane rh holds all 32 rows of column 2 cp + rh, written
  // as one 32-byte store
  uint32_t c8[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t got = __shfl_xor_sync(0xffffffffu, rh ? o0[j] : o1[j], 1);
    c8[j] = rh ? got : o0[j];          // rows 4 j .. 4 j + 3
    c8[4 + j] = rh ? o1[j] : got;      // rows 16 + 4 j .. 16 + 4 j + 3
  }
  stg32(q_c_blk + (int64_t)(2 * cp + rh) * rp, c8);
  at_c[atom_byte(c0 + 2 * cp + rh, tb)] = live ? (uint8_t)((rh ? ex1 : ex0) + 127) : (uint8_t)0x7F;
  __syncwarp();  // s_tr is read before the next block writes it
}

// ------------------------------------------------------------ tile decode
struct TileInfo {
  int g, m0, n0, rows, nkb, kbase, klast;
  int split, nsplit, kst;  // GROUP_K: K range j of nsplit, its first 128-row stage in the group
};

// K ranges of a weight-gradient group of c rows cut at threshold kc: ns ranges of ck rows
// (ck a multiple of 128, the last range shorter); ns = 1 when c <= kc or kc == 0.
__host__ __device__ __forceinline__ void wgrad_split(int c, int kc, int& ns, int& ck) {
  if (kc <= 0 || c <= kc) { ns = 1; ck = c; return; }
  const int n0 = (c + kc - 1) / kc;
  ck = (((c + n0 - 1) / n0) + 127) & ~127;
  ns = (c + ck - 1) / ck;
}

// GROUP_K with s_stg (MXFP8 weight gradients): the operands' token axis is stage-padded,
// every expert's tokens starting a 128-row stage (stage prefix s_stg) and the rows past
// its last token holding zero codes, so K runs over whole stages and nothing is zeroed.
template <int BN, int EPI, bool GROUP_K, int TM = BM, int KE = BK>
__device__ __forceinline__ TileInfo decode_tile(int t, const GemmParams& p, const int* s_off,
                                                const int* s_pre, int nN,
                                                const int* s_stg = nullptr) {
  TileInfo ti;
  if constexpr (GROUP_K) {
    const int per = (p.M / TM) * nN;
    int g, local;
    if (p.kchunk) {  // tile prefix over groups (ranges x per)
      int lo = 0, hi = p.E - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pre[mid] <= t) lo = mid; else hi = mid - 1;
      }
      g = lo;
      local = t - s_pre[g];
    } else {
      g = t / per;
      local = t - g * per;
    }
    const int j = local / per, rem = local - j * per;
    ti.g = g;
    ti.m0 = (rem / nN) * TM;
    ti.n0 = (rem % nN) * BN;
    ti.rows = TM;
    const int k0 = s_off[g], kg = s_off[g + 1] - k0;
    int ns, ck;
    wgrad_split(kg, p.kchunk, ns, ck);
    const int kb0 = j * ck, kn = min(ck, kg - kb0);
    ti.split = j;
    ti.nsplit = ns;
    ti.kst = kb0 / 128;
    ti.kbase = (s_stg ? s_stg[g] * 128 : k0) + kb0;
    ti.nkb = (kn + KE - 1) / KE;
    ti.klast = s_stg ? KE : kn - (ti.nkb - 1) * KE;
  } else {
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {  // last expert whose tile prefix is <= t (skips empty experts)
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    ti.g = lo;
    const int local = t - s_pre[lo];
    const int mt = local / nN, nt = local - mt * nN;
    ti.m0 = s_off[lo] + mt * TM;
    ti.rows = min(TM, s_off[lo + 1] - s_off[lo] - mt * TM);
    ti.n0 = nt * (EPI == EPI_SWIGLU_FWD ? BN / 2 : BN);
    ti.kbase = lo * p.b_rows;
    ti.nkb = p.K / KE;
    ti.klast = KE;
    ti.split = 0;
    ti.nsplit = 1;
    ti.kst = 0;
  }
  return ti;
}

// ------------------------------------------------------------------ kernel
template <int BN, bool A_MN, bool B_MN, int EPI, bool GROUP_K, bool PAIR = false, bool FP8 = false>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_sm100(const __grid_constant__ GemmParams p) {
  using C = Cfg<BN, PAIR, EPI, FP8>;
  const uint64_t wl = p.wait_ns ? p.wait_ns : (uint64_t)MOE_WAIT_NS;  // bounded-wait limit
  static_assert(!FP8 || ((BN == 128 || BN == 256) && (!PAIR || BN == 256)),
                "MXFP8 tiles: 128 x 128 or 128 x 256, or 256 x 256 on a CTA pair");
  static_assert(!FP8 || EPI != EPI_SWIGLU_FWD || BN == 256, "MXFP8 SwiGLU tiles pair 128 gate with 128 up columns");
  // epilogue warps 6..9 idle when a thread must hold a whole row (router)
  constexpr bool kHalfIdle = EPI == EPI_ROUTER;
  constexpr int S = C::kStages;
  static_assert(EPI != EPI_SWIGLU_FWD || BN == 256, "SwiGLU forward pairs 128 gate with 128 up columns");
  static_assert(!PAIR || (BN == 256 && !A_MN && EPI != EPI_ROUTER && (!GROUP_K || FP8)),
                "CTA pairs serve the row-grouped GEMMs with N = 256 and the MXFP8 weight gradients");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStage);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_off = reinterpret_cast<int*>(smem + C::kOffSoff);
  int* s_pre = s_off + 1025;
  int* s_sel = reinterpret_cast<int*>(smem + C::kOffSel);  // EPI_ROUTER: [4][256] histogram
  // GROUP_K: s_pre = tile prefix (split groups), s_stg = MXFP8 128-row stage prefix (in the
  // router histogram area), s_slot = partial-slot prefix
  int* s_stg = s_sel;
  int* s_slot = reinterpret_cast<int*>(smem + C::kOffExtra);
  uint8_t* s_store = smem + C::kOffStore;                   // TMA-store staging

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  // PAIR: the two CTAs of a cluster (ranks 0 and 1) share every tile; rank 0 (the
  // leader) issues the MMAs for both.
  const uint32_t rank = PAIR ? cluster_rank() : 0;
  const bool leader = rank == 0;
  const int tile0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tstride = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int nN = GROUP_K ? p.N / BN
                         : (EPI == EPI_SWIGLU_FWD ? p.N / (BN / 2) : (EPI == EPI_ROUTER ? 1 : p.N / BN));

  for (int g = threadIdx.x; g <= E; g += kThreads)
    s_off[g] = p.offsets ? p.offsets[g]
                         : (GROUP_K ? min(g * p.split, p.rows_total) : (g == 0 ? 0 : p.rows_total));
  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
      for (int a = 0; a < 2; ++a) {
        mbar_init(&tfull[a], 1);
        mbar_init(&tempty[a], PAIR ? 2 * (kThreads - 64) : (kHalfIdle ? 128 : kThreads - 64));
      }
      mbar_init(drain, 1);
      *s_abort = 0;
      fence_mbar_init();
    }
    __syncwarp();
    if constexpr (PAIR) tmem_alloc_pair(s_tmem, C::kTmemCols);
    else tmem_alloc(s_tmem, C::kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the peer's barriers exist before anyone signals them
  if constexpr (!GROUP_K) {
    if (warp == 1) {  // per-expert tile prefix (E <= 1024: 32 experts per lane)
      const int lo = lane * 32, hi = min(lo + 32, E);
      int s = 0;
      for (int g = lo; g < hi; ++g) s += ((s_off[g + 1] - s_off[g] + C::kTileM - 1) / C::kTileM) * nN;
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      int run = incl - s;
      for (int g = lo; g < hi; ++g) {
        s_pre[g] = run;
        run += ((s_off[g + 1] - s_off[g] + C::kTileM - 1) / C::kTileM) * nN;
      }
      if (lane == 31) s_pre[E] = incl;
      if constexpr (FP8 && PAIR) {
        // the A scale atoms are numbered per 128-row tile of each expert
        int s1 = 0;
        for (int g = lo; g < hi; ++g) s1 += (s_off[g + 1] - s_off[g] + BM - 1) / BM;
        int incl1 = s1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, incl1, o);
          if (lane >= o) incl1 += n;
        }
        int run1 = incl1 - s1;
        for (int g = lo; g < hi; ++g) {
          s_sel[g] = run1;
          run1 += (s_off[g + 1] - s_off[g] + BM - 1) / BM;
        }
      }
    }
  }
  if constexpr (GROUP_K) {
    // per-group prefixes, 32 groups per lane of warp 1 (E <= 1024): tiles (split groups),
    // partial slots (groups cut into several K ranges) and MXFP8 128-row stages
    if (warp == 1 && (p.kchunk || FP8)) {
      const int per = (p.M / C::kTileM) * nN;
      const int lo = lane * 32, hi = min(lo + 32, E);
      int st = 0, sl = 0, sg = 0;
      for (int g = lo; g < hi; ++g) {
        const int c = s_off[g + 1] - s_off[g];
        int ns, ck;
        wgrad_split(c, p.kchunk, ns, ck);
        st += ns * per;
        sl += ns > 1 ? ns : 0;
        sg += (c + 127) / 128;
      }
      int it_ = st, il = sl, ig = sg;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, it_, o);
        const int b = __shfl_up_sync(0xffffffffu, il, o);
        const int c = __shfl_up_sync(0xffffffffu, ig, o);
        if (lane >= o) { it_ += a; il += b; ig += c; }
      }
      int rt = it_ - st, rl = il - sl, rg = ig - sg;
      for (int g = lo; g < hi; ++g) {
        const int c = s_off[g + 1] - s_off[g];
        int ns, ck;
        wgrad_split(c, p.kchunk, ns, ck);
        s_pre[g] = rt;
        s_slot[g] = rl;
        s_stg[g] = rg;
        rt += ns * per;
        rl += ns > 1 ? ns : 0;
        rg += (c + 127) / 128;
      }
      if (lane == 31) s_pre[E] = it_;
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = GROUP_K ? (p.kchunk ? s_pre[E] : E * (p.M / C::kTileM) * nN) : s_pre[E];

  auto fail = [&]() {
    record_status(p.status, MOE_ERR_TIMEOUT);
    *s_abort = 1;
  };
  // this CTA's share of tile t (a pair splits the 256 rows 128 / 128)
  auto decode = [&](int t) {
    TileInfo ti = decode_tile<BN, EPI, GROUP_K, C::kTileM, C::kBKe>(t, p, s_off, s_pre, nN,
                                                                     GROUP_K && FP8 ? s_stg : nullptr);
    if constexpr (PAIR) {
      ti.m0 += BM * (int)rank;
      ti.rows = max(0, min(BM, ti.rows - BM * (int)rank));
    }
    return ti;
  };

  if (warp == 0 && FP8) {
    // ---------------------------------------------------- producer (MXFP8)
    // Per stage: the A and B tiles by TMA and their two 512-byte scale atoms by bulk
    // copy, all completing on the stage's full barrier.  Atom order in global memory:
    //   row-grouped A (K-major):   (M tile over all experts) * K/128 + k stage
    //   K-major B (weights):       (expert * N tiles + n tile) * K/128 + k stage
    //   MN-major B (weights):      (expert * K/128 + k stage) * N/128 + n tile
    //   GROUP_K A and B:           (k stage over all groups) * (M or N)/128 + tile
    if (lane == 0) {
      tma_prefetch_desc(&p.tmA);
      tma_prefetch_desc(&p.tmB);
      uint32_t it = 0;
      int s = 0;
      uint32_t ph = 1;  // the first pass over the ring finds every stage free
      bool ok = true;
      const int kq = GROUP_K ? 0 : p.K / C::kBKe;
      const uint32_t leader_full = PAIR ? map_to_rank(&full[0], 0) : 0;
      for (int t = tile0; t < total && ok; t += tstride) {
        if (*s_abort) { ok = false; break; }
        const TileInfo ti = decode(t);
        const uint8_t* atomA;
        const uint8_t* atomB;
        // atomB2: the second B atom of a 256-wide tile (K-major B only; MN-major atoms
        // of one stage are adjacent and travel in one copy)
        const uint8_t* atomB2 = nullptr;
        if constexpr (GROUP_K) {
          const int64_t stage0 = s_stg[ti.g] + ti.kst;
          atomA = p.sfa + (stage0 * (p.M / BM) + ti.m0 / BM) * 512;
          atomB = p.sfb + (stage0 * (p.N / 128) + ti.n0 / 128) * 512;
        } else {
          const int mt = s_pre[ti.g] / nN + (ti.m0 - s_off[ti.g]) / BM;
          atomA = p.sfa + (int64_t)mt * kq * 512;
          if constexpr (!B_MN) {
            // K-major weights: atom (expert row tile) * K/128 + k stage, 128 rows per tile
            const int ntiles = p.b_rows / 128;
            if constexpr (EPI == EPI_SWIGLU_FWD && BN == 256) {
              atomB = p.sfb + ((int64_t)ti.g * ntiles + ti.n0 / 128) * kq * 512;
              atomB2 = p.sfb + ((int64_t)ti.g * ntiles + (p.f + ti.n0) / 128) * kq * 512;
            } else {
              atomB = p.sfb + ((int64_t)ti.g * ntiles + ti.n0 / 128) * kq * 512;
              if constexpr (BN == 256) atomB2 = atomB + (int64_t)kq * 512;
            }
          } else {
            atomB = p.sfb + ((int64_t)ti.g * kq * (p.N / 128) + ti.n0 / 128) * 512;
          }
        }
        // CTA pairs: atom indices (the atom tensors' row is twice the index).  A: this CTA's
        // 128-row tile of its expert; B: both 128-column halves of the tile.
        int64_t pa0 = 0, pb0 = 0, pb1 = 0;
        if constexpr (PAIR && !GROUP_K) {
          pa0 = ((int64_t)s_sel[ti.g] + (ti.m0 - s_off[ti.g]) / BM) * kq;
          if constexpr (!B_MN) {
            const int ntiles = p.b_rows / 128;
            // SwiGLU: the gate and the up row tiles; otherwise two adjacent row tiles
            const int t0 = ti.n0 / 128;
            const int t1 = EPI == EPI_SWIGLU_FWD ? (p.f + ti.n0) / 128 : ti.n0 / 128 + 1;
            pb0 = ((int64_t)ti.g * ntiles + t0) * kq;
            pb1 = ((int64_t)ti.g * ntiles + t1) * kq;
          } else {
            pb0 = (int64_t)ti.g * kq * (p.N / 128) + ti.n0 / 128;
            pb1 = pb0 + 1;
          }
        }
        for (int kb = 0; kb < ti.nkb; ++kb, ++it, s = (s + 1 == S ? 0 : s + 1), ph ^= (s == 0)) {
          if (!mbar_wait(&empty[s], ph, wl)) { fail(); ok = false; break; }
          if (!PAIR && p.drop_it && blockIdx.x == 0 && it + 1 == (uint32_t)p.drop_it) continue;  // test hook
          uint8_t* sa = smem + s * C::kStage;
          uint8_t* sb = sa + kABytes;
          uint8_t* sf = sb + C::kBBytes;
          const int kc = kb * C::kBKe;  // first K element of the stage
          if constexpr (PAIR) {
            // every load of both CTAs completes on the leader's barrier; only the leader arrives
            if (leader) mbar_arrive_expect_tx(&full[s], 2 * (kABytes + C::kBBytes + C::kSfLoad));
            const uint32_t bar = leader_full + 8 * s;
            if constexpr (GROUP_K) {
              // weight gradients (256 x 256 tiles): this CTA's 128 A rows and 128 of the
              // 256 B rows, K-major over the stage-padded token axis; the A atom of its
              // rows and both B atoms of the stage
              const int64_t zk = (int64_t)s_stg[ti.g] + ti.kst + kb;
              const int64_t ia = zk * (p.M / BM) + ti.m0 / BM;
              const int64_t ib = zk * (p.N / 128) + ti.n0 / 128;
              tma_load_2d_pair(sa, &p.tmA, ti.kbase + kc, ti.m0, bar);
              tma_load_2d_pair(sb, &p.tmB, ti.kbase + kc, ti.n0 + 128 * (int)rank, bar);
              tma_load_2d_pair(sf, &p.tmSfa, 0, (int)(2 * ia), bar);
              tma_load_2d_pair(sf + 512, &p.tmSfb, 0, (int)(2 * ib), bar);
              tma_load_2d_pair(sf + 1024, &p.tmSfb, 0, (int)(2 * ib + 2), bar);
              continue;
            }
            tma_load_2d_pair(sa, &p.tmA, kc, ti.m0, bar);
            if constexpr (!B_MN) {
              const int row = ti.kbase + (EPI == EPI_SWIGLU_FWD ? (rank == 0 ? ti.n0 : p.f + ti.n0)
                                                               : ti.n0 + 128 * (int)rank);
              tma_load_2d_pair(sb, &p.tmB, kc, row, bar);
            } else {
              tma_load_2d_pair(sb, &p.tmB, ti.n0 + 128 * (int)rank, ti.kbase + kc, bar);
            }
            // MN-major B atoms of one stage are N/128 apart in k; K-major ones 1 apart
            const int64_t bstep = B_MN ? (int64_t)kb * (p.N / 128) : (int64_t)kb;
            tma_load_2d_pair(sf, &p.tmSfa, 0, (int)(2 * (pa0 + kb)), bar);
            tma_load_2d_pair(sf + 512, &p.tmSfb, 0, (int)(2 * (pb0 + bstep)), bar);
            tma_load_2d_pair(sf + 1024, &p.tmSfb, 0, (int)(2 * (pb1 + bstep)), bar);
            continue;
          }
          constexpr uint32_t kSfB = (BN / 128) * 512;
          mbar_arrive_expect_tx(&full[s], kABytes + C::kBBytes + 512 + kSfB);
          if constexpr (GROUP_K) {
            // weight gradients: A and B K-major over the stage-padded token axis
            static_assert(!FP8 || (!A_MN && !B_MN), "MXFP8 weight-gradient operands are K-major");
            tma_load_2d(sa, &p.tmA, ti.kbase + kc, ti.m0, &full[s]);
#pragma unroll
            for (int i = 0; i < BN / 128; ++i)
              tma_load_2d(sb + i * 16384, &p.tmB, ti.kbase + kc, ti.n0 + 128 * i, &full[s]);
          } else if constexpr (!A_MN) {
            tma_load_2d(sa, &p.tmA, kc, ti.m0, &full[s]);
          } else {
            tma_load_2d(sa, &p.tmA, ti.m0, ti.kbase + kc, &full[s]);
          }
          if constexpr (!GROUP_K && !B_MN) {
            // boxes of BN/2 rows (SwiGLU: gate rows, then up rows) or of 128 rows
            if constexpr (EPI == EPI_SWIGLU_FWD) {
              tma_load_2d(sb, &p.tmB, kc, ti.kbase + ti.n0, &full[s]);
              tma_load_2d(sb + (BN / 2) * 128, &p.tmB, kc, ti.kbase + p.f + ti.n0, &full[s]);
            } else {
#pragma unroll
              for (int i = 0; i < BN / 128; ++i)
                tma_load_2d(sb + i * 16384, &p.tmB, kc, ti.kbase + ti.n0 + 128 * i, &full[s]);
            }
          } else if constexpr (!GROUP_K) {
#pragma unroll
            for (int i = 0; i < BN / 128; ++i)
              tma_load_2d(sb + i * 16384, &p.tmB, ti.n0 + 128 * i, ti.kbase + kc, &full[s]);
          }
          if constexpr (GROUP_K) {
            bulk_load(sf, atomA + (int64_t)kb * (p.M / BM) * 512, 512, &full[s]);
            bulk_load(sf + 512, atomB + (int64_t)kb * (p.N / 128) * 512, kSfB, &full[s]);
          } else if constexpr (B_MN) {
            bulk_load(sf, atomA + kb * 512, 512, &full[s]);
            bulk_load(sf + 512, atomB + (int64_t)kb * (p.N / 128) * 512, kSfB, &full[s]);
          } else {
            bulk_load(sf, atomA + kb * 512, 512, &full[s]);
            bulk_load(sf + 512, atomB + kb * 512, 512, &full[s]);
            if constexpr (BN == 256) bulk_load(sf + 1024, atomB2 + kb * 512, 512, &full[s]);
          }
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; ++j)
          (void)mbar_wait(&full[j % S], (j / S) & 1, wl);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tmA);
      tma_prefetch_desc(&p.tmB);
      uint32_t it = 0;
      int s = 0;
      uint32_t ph = 1;  // the first pass over the ring finds every stage free
      bool ok = true;
      const uint32_t leader_full = PAIR ? map_to_rank(&full[0], 0) : 0;
      for (int t = tile0; t < total && ok; t += tstride) {
        if (*s_abort) { ok = false; break; }
        const TileInfo ti = decode(t);
        for (int kb = 0; kb < ti.nkb; ++kb, ++it, s = (s + 1 == S ? 0 : s + 1), ph ^= (s == 0)) {
          if (!mbar_wait(&empty[s], ph, wl)) { fail(); ok = false; break; }
          if (!PAIR && p.drop_it && blockIdx.x == 0 && it + 1 == (uint32_t)p.drop_it) continue;  // test hook
          uint8_t* sa = smem + s * C::kStage;
          uint8_t* sb = sa + kABytes;
          const int kc = kb * BK;
          if constexpr (PAIR) {
            // both CTAs' bytes complete on the leader's barrier; only the leader arrives
            if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::kStage);
            const uint32_t bar = leader_full + 8 * s;
            tma_load_2d_pair(sa, &p.tmA, kc, ti.m0, bar);
            if constexpr (!B_MN) {
              const int row = ti.kbase + (EPI == EPI_SWIGLU_FWD ? (rank == 0 ? ti.n0 : p.f + ti.n0)
                                                               : ti.n0 + 128 * (int)rank);
              tma_load_2d_pair(sb, &p.tmB, kc, row, bar);
            } else {
#pragma unroll
              for (int i = 0; i < 2; ++i)
                tma_load_2d_pair(sb + i * 8192, &p.tmB, ti.n0 + 128 * (int)rank + 64 * i, ti.kbase + kc, bar);
            }
            continue;
          }
          mbar_arrive_expect_tx(&full[s], C::kStage);
          if constexpr (!A_MN) {
            tma_load_2d(sa, &p.tmA, kc, ti.m0, &full[s]);
          } else {
#pragma unroll
            for (int i = 0; i < 2; ++i) tma_load_2d(sa + i * 8192, &p.tmA, ti.m0 + 64 * i, ti.kbase + kc, &full[s]);
          }
          if constexpr (!B_MN) {
            constexpr int kBox = C::kBoxRows;
#pragma unroll
            for (int i = 0; i < BN / kBox; ++i) {
              const int row = ti.kbase + (EPI == EPI_SWIGLU_FWD ? (i == 0 ? ti.n0 : p.f + ti.n0)
                                                               : ti.n0 + kBox * i);
              tma_load_2d(sb + i * kBox * 128, &p.tmB, kc, row, &full[s]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i)
              tma_load_2d(sb + i * 8192, &p.tmB, ti.n0 + 64 * i, ti.kbase + kc, &full[s]);
          }
        }
      }
      if (!ok && leader) {  // let the loads in flight land before shared memory is released
        for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; ++j)
          (void)mbar_wait(&full[j % S], (j / S) & 1, wl);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // One thread issues.  Its per-stage work is kept small, since at these tile sizes
    // the issuing thread, not the tensor core, sets the pace: the ring position and the
    // barrier parity advance incrementally, and a stage's shared-memory descriptors are
    // the ring's base descriptors plus constants (the start-address field counts 16-byte
    // units, and no start address of the ring reaches 2^18 bytes).
    constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)A_MN << 15) |
                               ((uint32_t)B_MN << 16) | ((uint32_t)(BN >> 3) << 17) |
                               ((uint32_t)(C::kTileM >> 4) << 24);
    constexpr uint32_t idesc_mx = ((uint32_t)A_MN << 15) | ((uint32_t)B_MN << 16) |
                                  ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(C::kTileM >> 4) << 24);
    // MN-major operands: LBO = distance between 64 (bf16) or 128 (fp8) element MN blocks
    constexpr uint32_t kLboA = A_MN ? (FP8 ? 16384 : 8192) : 16;
    constexpr uint32_t kLboB = B_MN ? (FP8 ? 16384 : 8192) : 16;
    // advance of the start field per MMA along K (K = 16 bf16 or 32 fp8 per MMA)
    constexpr uint32_t kStepA = (A_MN ? (FP8 ? 4096 : 2048) : 32) >> 4;
    constexpr uint32_t kStepB = (B_MN ? (FP8 ? 4096 : 2048) : 32) >> 4;
    constexpr uint32_t kStageU = C::kStage >> 4;
    const uint32_t ring = smem_u32(smem);
    const uint64_t desc_a0 = sdesc(ring, kLboA, 1024);
    const uint64_t desc_b0 = sdesc(ring + kABytes, kLboB, 1024);
    const uint64_t desc_f0 = sf_desc(ring + kABytes + C::kBBytes);
    uint32_t it = 0, acc_it = 0;
    int stg = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = tile0; t < total && ok && leader; t += tstride) {
      if (__any_sync(0xffffffffu, *s_abort)) { ok = false; break; }
      const TileInfo ti = decode(t);
      const int acc = C::kAccBufs == 2 ? (int)(acc_it & 1) : 0;
      const uint32_t acc_ph = C::kAccBufs == 2 ? (acc_it >> 1) & 1 : acc_it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&tempty[acc], acc_ph ^ 1, wl))) {
        if (lane == 0) fail();
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < ti.nkb; ++kb, ++it) {
        bool w = true;
        if (lane == 0) w = mbar_wait(&full[stg], ph, wl);
        if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
          if (lane == 0) fail();
          ok = false;
          break;
        }
        tc_fence_after();
        if constexpr (GROUP_K) {
          if (kb == ti.nkb - 1 && ti.klast < C::kBKe) {
            // Rows [klast, K rows of a box) of every box hold the next expert's tokens:
            // zero them.  bf16 boxes are 64 M/N x 64 K rows (8 KB), fp8 boxes 128 x 128 (16 KB).
            uint8_t* sa = smem + stg * C::kStage;
            uint8_t* sb = sa + kABytes;
            constexpr int kBoxRowsK = C::kBKe;
            constexpr int kBoxBytes = kBoxRowsK * 128;
            constexpr int kABoxes = kABytes / kBoxBytes;
            constexpr int kBoxes = kABoxes + C::kBBytes / kBoxBytes;
            // The rows are 128 bytes each, so the tail of a box is one contiguous range
            // (the 128-byte swizzle only permutes 16-byte pieces within a row).
            const int tail = (kBoxRowsK - ti.klast) * 128;
#pragma unroll
            for (int box = 0; box < kBoxes; ++box) {
              uint8_t* z = (box < kABoxes ? sa + box * kBoxBytes : sb + (box - kABoxes) * kBoxBytes) +
                           ti.klast * 128;
              for (int o = lane * 16; o < tail; o += 512)
                *reinterpret_cast<uint4*>(z + o) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t so = (uint32_t)stg * kStageU;
          const uint64_t ad = desc_a0 + so, bd = desc_b0 + so;
          if constexpr (FP8) {
            // scales of this stage -> TMEM, then four K = 32 block-scaled MMAs.  The
            // scale slots rotate over 4 x 16 TMEM columns; the scales of B atom i (rows
            // 128 i ..) sit 4 i columns after the first.
            const uint32_t tsf = tmem_base + C::kSfCol + 16 * (it & (C::kSfSlots - 1));
            if constexpr (PAIR) {
              // each CTA copies its own atoms into its own TMEM; the leader's MMAs then
              // read both CTAs' A rows, B halves and scales
              tmem_cp_sf_pair(tsf, desc_f0 + so);
#pragma unroll
              for (int i = 0; i < 2; ++i)
                tmem_cp_sf_pair(tsf + 4 + 4 * i, desc_f0 + so + ((512 + 512 * i) >> 4));
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_mxf8_pair(d_tmem, ad + k * kStepA, bd + k * kStepB,
                               idesc_mx | ((uint32_t)k << 4) | ((uint32_t)k << 29), (kb | k) != 0,
                               tsf | ((uint32_t)k << 30), (tsf + 4) | ((uint32_t)k << 30));
              umma_commit_pair(&empty[stg]);
            } else {
              tmem_cp_sf(tsf, desc_f0 + so);
#pragma unroll
              for (int i = 0; i < BN / 128; ++i)
                tmem_cp_sf(tsf + 4 + 4 * i, desc_f0 + so + ((512 + 512 * i) >> 4));
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_mxf8(d_tmem, ad + k * kStepA, bd + k * kStepB,
                          idesc_mx | ((uint32_t)k << 4) | ((uint32_t)k << 29), (kb | k) != 0,
                          tsf | ((uint32_t)k << 30), (tsf + 4) | ((uint32_t)k << 30));
              umma_commit(&empty[stg]);
            }
          } else {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              if constexpr (PAIR) umma_bf16_pair(d_tmem, ad + k * kStepA, bd + k * kStepB, idesc, (kb | k) != 0);
              else umma_bf16(d_tmem, ad + k * kStepA, bd + k * kStepB, idesc, (kb | k) != 0);
            }
            if constexpr (PAIR) umma_commit_pair(&empty[stg]);
            else umma_commit(&empty[stg]);
          }
        }
        if (++stg == S) { stg = 0; ph ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) {
        if constexpr (PAIR) umma_commit_pair(&tfull[acc]);
        else umma_commit(&tfull[acc]);
      }
      __syncwarp();
      ++acc_it;
    }
    if (!ok && lane == 0) {  // wait for this thread's MMAs before TMEM is freed
      if constexpr (PAIR) umma_commit_pair(drain);
      else umma_commit(drain);
      (void)mbar_wait(drain, 0, wl);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Eight warps: two per TMEM lane quarter (warp % 4), each taking half of
    // the tile's 32-column chunks.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    constexpr int kChunks = (EPI == EPI_SWIGLU_FWD ? BN / 2 : BN) / 32;
    constexpr int kMine = kChunks / 2;
    const int c0 = half * kMine;
    uint32_t acc_it = 0;
    // this warp's TMA-store staging: two 2 KB slots (bf16 outputs) or one (fp32 wgrad)
    constexpr size_t kWarpStore = C::kStoreBytes / 8;
    static_assert(EPI == EPI_ROUTER || EPI == EPI_ROUTER_DX ||
                      kWarpStore >= (EPI == EPI_WGRAD ? 2048 : 4096),
                  "staging slots of an epilogue warp fit its share of the store area");
    uint8_t* wbuf = s_store + (warp - 2) * kWarpStore;
    uint32_t slot = 0;
    // The router epilogue keeps a whole logit row per thread: warps 2..5 only.
    const bool idle = kHalfIdle && half == 1;
    const uint32_t leader_tempty = PAIR ? map_to_rank(&tempty[0], 0) : 0;
    for (int t = tile0; t < total && !idle; t += tstride) {
      if (__any_sync(0xffffffffu, *s_abort)) break;
      const TileInfo ti = decode(t);
      const int acc = C::kAccBufs == 2 ? (int)(acc_it & 1) : 0;
      const uint32_t acc_ph = C::kAccBufs == 2 ? (acc_it >> 1) & 1 : acc_it & 1;
      const bool valid = row < ti.rows;
      // SwiGLU backward: a and u of the first chunk do not depend on the
      // accumulator, so their loads are in flight while the main loop runs.
      uint32_t av[16], uv[16];
      const __nv_bfloat16* arow = nullptr;
      if constexpr (EPI == EPI_SWIGLU_BWD) {
        arow = p.act + (int64_t)(ti.m0 + row) * p.ld_act;
        if (valid) load_au(arow, ti.n0 + c0 * 32, p.f, av, uv);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_ph, wl))) {
        fail();
        break;
      }
      tc_fence_after();
      const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      auto release = [&]() {
        tc_fence_before();
        if constexpr (PAIR) mbar_arrive_remote(leader_tempty + 8 * acc);
        else mbar_arrive(&tempty[acc]);
      };
      // rows of this CTA's tile that a box starting at tile row b0 may write
      auto box_valid = [&](int b0) { return max(0, min(16, ti.rows - b0)); };
      const int grow0 = ti.m0 + q * 32;  // first global row of this warp
      if constexpr (EPI == EPI_SWIGLU_FWD) {
        // 64 gate columns per warp (two chunks): a, u, h as three boxes per row half
        uint32_t pa[32], pu[32], ph[32];
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
          const int c = c0 + ci;
          uint32_t g[32], u[32];
          tmem_ld32(ta + c * 32, g);
          tmem_ld32(ta + BN / 2 + c * 32, u);
          tmem_wait_ld();
          tmem_tie(g);
          tmem_tie(u);
          if (ci == 1) release();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = __uint_as_float(g[2 * i]), a1 = __uint_as_float(g[2 * i + 1]);
            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
            pa[16 * ci + i] = pack_bf16(a0, a1);
            pu[16 * ci + i] = pack_bf16(u0, u1);
            ph[16 * ci + i] = pack_bf16(a0 * sigmoidf_(a0) * u0, a1 * sigmoidf_(a1) * u1);
          }
        }
        const int col = ti.n0 + c0 * 32;
        __nv_bfloat16* arow = p.out + (int64_t)(ti.m0 + row) * p.ld_out;
        if constexpr (FP8) {
          if (p.mx_q_r && ti.rows > 0) {
            // h (the down GEMM's operand) also leaves as its two MXFP8 copies: this warp's 32
            // rows are one 32-token block and its tile a stage, as for [da | du].  Its
            // shared-memory scratch is the warp's store staging: the stores that read it
            // finish first.
            if (lane == 0) tma_store_wait_read();
            __syncwarp();
            const int stage = (PAIR ? s_sel[ti.g] : s_pre[ti.g] / nN) + (ti.m0 - s_off[ti.g]) / BM;
            const int kq = p.f / 128;
            const int64_t grow = ti.m0 + row;
#pragma unroll
            for (int ci = 0; ci < 2; ++ci) {
              const int gc = col + 32 * ci;  // column of h
              mx_emit_block(ph + 16 * ci, valid, q * 32 < ti.rows, p.mx_q_r + grow * p.f + gc,
                            p.mx_s_r + ((int64_t)stage * kq + gc / 128) * 512 +
                                atom_byte(row, (gc & 127) >> 5),
                            p.mx_q_c + (int64_t)gc * p.mx_rp + 128 * (int64_t)stage + 32 * q,
                            p.mx_rp, p.mx_s_c + ((int64_t)stage * kq + gc / 128) * 512, gc & 96,
                            q, reinterpret_cast<uint32_t*>(wbuf));
            }
          }
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int vr = box_valid(q * 32 + 16 * hh);
          put_box_bf16(wbuf, slot, &p.tmOut, pa, hh, col, grow0 + 16 * hh, vr, arow + col);
          put_box_bf16(wbuf, slot, &p.tmOut, pu, hh, p.f + col, grow0 + 16 * hh, vr, arow + p.f + col);
          put_box_bf16(wbuf, slot, &p.tmOut, ph, hh, 2 * p.f + col, grow0 + 16 * hh, vr, arow + 2 * p.f + col);
        }
      } else if constexpr (EPI == EPI_STORE) {
        // every chunk of this warp is read (and packed to bf16) before the accumulator is
        // released, so that the next tile's MMAs overlap the stores
        __nv_bfloat16* orow = p.out + (int64_t)(ti.m0 + row) * p.ld_out;
        uint32_t pk[kMine / 2][32];
#pragma unroll
        for (int pc = 0; pc < kMine / 2; ++pc) {
#pragma unroll
          for (int ci = 0; ci < 2; ++ci) {
            uint32_t v[32];
            tmem_ld32(ta + (c0 + 2 * pc + ci) * 32, v);
            tmem_wait_ld();
            tmem_tie(v);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[pc][16 * ci + i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          }
        }
        release();
#pragma unroll
        for (int pc = 0; pc < kMine / 2; ++pc) {
          const int col = ti.n0 + (c0 + 2 * pc) * 32;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            put_box_bf16(wbuf, slot, &p.tmOut, pk[pc], hh, col, grow0 + 16 * hh,
                         box_valid(q * 32 + 16 * hh), orow + col);
        }
      } else if constexpr (EPI == EPI_SWIGLU_BWD) {
        __nv_bfloat16* drow = p.out + (int64_t)(ti.m0 + row) * p.ld_out;
        // A single accumulator (256-wide MXFP8 tiles) would stay busy through this warp's
        // loads of a and u and its stores, holding back the next tile's MMAs.  Instead its
        // chunks 1..3 are parked in the spare TMEM columns and chunk 0 is kept in registers,
        // so the accumulator is released at once.
        constexpr bool kPark = C::kAccBufs == 1;
        static_assert(!kPark || (kMine == 4 && C::kSpareCol + 2 * 96 <= 512),
                      "three parked chunks per warp fit after the scale slots");
        uint32_t v0[32];
        const uint32_t tsp = tmem_base + ((uint32_t)(q * 32) << 16) + C::kSpareCol + half * 96;
        if constexpr (kPark) {
#pragma unroll
          for (int i = 1; i < kMine; ++i) {
            uint32_t t[32];
            tmem_ld32(ta + (c0 + i) * 32, t);
            tmem_wait_ld();
            tmem_tie(t);
            tmem_st32(tsp + (i - 1) * 32, t);
          }
          tmem_ld32(ta + c0 * 32, v0);
          tmem_wait_ld();
          tmem_tie(v0);
          tmem_wait_st();
          release();
        }
#pragma unroll
        for (int pc = 0; pc < kMine / 2; ++pc) {
          uint32_t pda[32], pdu[32];
#pragma unroll
          for (int ci = 0; ci < 2; ++ci) {
            const int cidx = 2 * pc + ci;  // chunk of this warp, 0 .. kMine-1
            const int col = ti.n0 + (c0 + cidx) * 32;
            uint32_t an[16], un[16];
            if (cidx + 1 < kMine && valid) load_au(arow, col + 32, p.f, an, un);  // one chunk ahead
            uint32_t v[32];
            if constexpr (kPark) {
              if (cidx == 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = v0[i];
              } else {
                tmem_ld32(tsp + (cidx - 1) * 32, v);
                tmem_wait_ld();
                tmem_tie(v);
              }
            } else {
              tmem_ld32(ta + (c0 + cidx) * 32, v);
              tmem_wait_ld();
              tmem_tie(v);
              if (cidx == kMine - 1) release();
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float da[2], du[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const float dh = __uint_as_float(v[2 * i + h]);
                const float a = h ? bf_hi(av[i]) : bf_lo(av[i]);
                const float u = h ? bf_hi(uv[i]) : bf_lo(uv[i]);
                const float sg = sigmoidf_(a);
                da[h] = dh * u * sg * (1.f + a * (1.f - sg));
                du[h] = dh * a * sg;
              }
              pda[16 * ci + i] = pack_bf16(da[0], da[1]);
              pdu[16 * ci + i] = pack_bf16(du[0], du[1]);
            }
            if (cidx + 1 < kMine) {
#pragma unroll
              for (int i = 0; i < 16; ++i) { av[i] = an[i]; uv[i] = un[i]; }
            }
          }
          const int col = ti.n0 + (c0 + 2 * pc) * 32;
          if constexpr (FP8) {
            if (p.mx_q_r) {
              // [da | du] as its MXFP8 operand copies: this warp's 32 rows are one 32-token
              // block (tiles and stages both start at every expert), and its tile is a stage
              if (ti.rows > 0) {
                const int stage = (PAIR ? s_sel[ti.g] : s_pre[ti.g] / nN) + (ti.m0 - s_off[ti.g]) / BM;
                const int kq = 2 * p.f / 128;
                uint32_t* s_tr = reinterpret_cast<uint32_t*>(wbuf);
                const int64_t grow = ti.m0 + row;
#pragma unroll
                for (int ci = 0; ci < 2; ++ci) {
#pragma unroll
                  for (int du_part = 0; du_part < 2; ++du_part) {
                    const int gc = (du_part ? p.f : 0) + col + 32 * ci;  // column of [da | du]
                    const uint32_t* pk = (du_part ? pdu : pda) + 16 * ci;
                    mx_emit_block(pk, valid, q * 32 < ti.rows, p.mx_q_r + grow * (2 * p.f) + gc,
                                  p.mx_s_r + ((int64_t)stage * kq + gc / 128) * 512 +
                                      atom_byte(row, (gc & 127) >> 5),
                                  p.mx_q_c + (int64_t)gc * p.mx_rp + 128 * (int64_t)stage + 32 * q,
                                  p.mx_rp, p.mx_s_c + ((int64_t)stage * kq + gc / 128) * 512,
                                  gc & 96, q, s_tr);
                  }
                }
              }
              if (p.out && valid) {
                uint32_t lo[16], hi[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) { lo[i] = pda[i]; hi[i] = pda[16 + i]; }
                store_64B(drow + col, lo);
                store_64B(drow + col + 32, hi);
#pragma unroll
                for (int i = 0; i < 16; ++i) { lo[i] = pdu[i]; hi[i] = pdu[16 + i]; }
                store_64B(drow + p.f + col, lo);
                store_64B(drow + p.f + col + 32, hi);
              }
              continue;
            }
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int vr = box_valid(q * 32 + 16 * hh);
            put_box_bf16(wbuf, slot, &p.tmOut, pda, hh, col, grow0 + 16 * hh, vr, drow + col);
            put_box_bf16(wbuf, slot, &p.tmOut, pdu, hh, p.f + col, grow0 + 16 * hh, vr, drow + p.f + col);
          }
        }
      } else if constexpr (EPI == EPI_ROUTER) {
        // logits (+ bias), softmax over the p.N experts, top-k (lowest index wins
        // ties), then this 128-token block's per-expert counts and in-block ranks.
        const int Er = p.N, k = p.topk;
        const int64_t tok = ti.m0 + row;
        float topv[kRouterKMax];
        int topi[kRouterKMax];
#pragma unroll
        for (int j = 0; j < kRouterKMax; ++j) { topv[j] = -INFINITY; topi[j] = -1; }
        float mx = -INFINITY;
        float* lrow = p.logits + tok * Er;
#pragma unroll 1
        for (int c = 0; c < BN / 16; ++c) {
          uint32_t v[16];
          tmem_ld16(ta + c * 16, v);
          tmem_wait_ld();
          tmem_tie16(v);
          float l[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = c * 16 + i;
            l[i] = e < Er ? __uint_as_float(v[i]) + (p.bias ? p.bias[e] : 0.f) : -INFINITY;
            if (e < Er) {
              mx = fmaxf(mx, l[i]);
              float cv = l[i];
              int ci = e;
#pragma unroll
              for (int j = 0; j < kRouterKMax; ++j) {  // ascending e: equal values keep the lower index
                if (j < k && (topi[j] < 0 || cv > topv[j])) {
                  const float tv = topv[j]; topv[j] = cv; cv = tv;
                  const int tix = topi[j]; topi[j] = ci; ci = tix;
                }
              }
            }
          }
          if (valid) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int e0 = c * 16 + 4 * q4;
              if ((Er & 3) == 0 && e0 + 4 <= Er)
                *reinterpret_cast<float4*>(lrow + e0) = make_float4(l[4 * q4], l[4 * q4 + 1], l[4 * q4 + 2], l[4 * q4 + 3]);
              else
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  if (e0 + i < Er) lrow[e0 + i] = l[4 * q4 + i];
            }
          }
        }
        float sum = 0.f;
#pragma unroll 1
        for (int c = 0; c < BN / 16; ++c) {
          uint32_t v[16];
          tmem_ld16(ta + c * 16, v);
          tmem_wait_ld();
          tmem_tie16(v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = c * 16 + i;
            if (e < Er) sum += expf(__uint_as_float(v[i]) + (p.bias ? p.bias[e] : 0.f) - mx);
          }
        }
        release();
        // block counts and in-block ranks: a per-warp histogram in shared memory
        // (integer atomics: the counts do not depend on their order) and, for the
        // rank, a count of the earlier lanes of this warp that picked the same expert
        int* cnt = s_sel;  // [4 row quarters][256 experts]
        const int wq = q;  // this warp's rows are 32 wq .. 32 wq + 31 of the tile
        for (int i = row; i < 4 * 256; i += 128) cnt[i] = 0;
#pragma unroll
        for (int j = 0; j < kRouterKMax; ++j) {
          if (j < k && valid) {
            p.topk_idx[tok * k + j] = topi[j];
            p.topk_gate[tok * k + j] = expf(topv[j] - mx) / sum;
          }
          if (!valid) topi[j] = -1;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
        for (int j = 0; j < kRouterKMax; ++j)
          if (j < k && valid) atomicAdd(&cnt[wq * 256 + topi[j]], 1);
        int rank[kRouterKMax];
#pragma unroll
        for (int j = 0; j < kRouterKMax; ++j) rank[j] = 0;
        for (int l = 0; l < 31; ++l) {
#pragma unroll
          for (int j2 = 0; j2 < kRouterKMax; ++j2) {
            if (j2 >= k) break;
            const int v = __shfl_sync(0xffffffffu, topi[j2], l);
            if (l < lane) {
#pragma unroll
              for (int j = 0; j < kRouterKMax; ++j) rank[j] += (v == topi[j]);
            }
          }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (valid) {
#pragma unroll
          for (int j = 0; j < kRouterKMax; ++j) {
            if (j < k) {
              int r = rank[j];
              for (int w2 = 0; w2 < wq; ++w2) r += cnt[w2 * 256 + topi[j]];
              p.localrank[tok * k + j] = r;
            }
          }
        }
        const int blk = ti.m0 / BM;
        for (int e = row; e < Er; e += 128)
          p.blockcounts[(int64_t)e * p.nb + blk] = cnt[e] + cnt[256 + e] + cnt[512 + e] + cnt[768 + e];
        asm volatile("bar.sync 1, 128;" ::: "memory");  // the histogram is reused by the next tile
      } else if constexpr (EPI == EPI_ROUTER_DX) {
        // router backward: dx = dl w_router (the accumulator) + the token's k expert rows
        // (no slot_row: one row per token, the token's own row of p.act)
        const int k = p.slot_row ? p.topk : 1;
        const int64_t tok = ti.m0 + row;
        int rj[kRouterKMax];
#pragma unroll
        for (int j = 0; j < kRouterKMax; ++j)
          rj[j] = (valid && j < k) ? (p.slot_row ? __ldg(p.slot_row + tok * k + j) : (int)tok) : -1;
        __nv_bfloat16* orow = p.out + tok * p.ld_out;
#pragma unroll
        for (int ci = 0; ci < kMine; ++ci) {
          const int col = ti.n0 + (c0 + ci) * 32;
          uint32_t v[32];
          tmem_ld32(ta + (c0 + ci) * 32, v);
          tmem_wait_ld();
          tmem_tie(v);
          if (ci == kMine - 1) release();
          if (valid) {
            float accf[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) accf[i] = __uint_as_float(v[i]);
#pragma unroll
            for (int j = 0; j < kRouterKMax; ++j) {
              if (rj[j] < 0) continue;
              const uint4* src = reinterpret_cast<const uint4*>(p.act + (int64_t)rj[j] * p.ld_act + col);
#pragma unroll
              for (int i4 = 0; i4 < 4; ++i4) {
                const uint4 w = __ldg(src + i4);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  accf[8 * i4 + 2 * h] += bf_lo(ww[h]);
                  accf[8 * i4 + 2 * h + 1] += bf_hi(ww[h]);
                }
              }
            }
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(accf[2 * i], accf[2 * i + 1]);
            store_64B(orow + col, pk);
          }
        }
      } else {  // EPI_WGRAD
        // a group cut into K ranges writes fp32 partial sums to its slot of `part`
        const bool partial = ti.nsplit > 1;
        const CUtensorMap* tmo = partial ? &p.tmPart : &p.tmOut;
        const int64_t orow0 = (partial ? (int64_t)(s_slot[ti.g] + ti.split) : (int64_t)ti.g) * p.M +
                              ti.m0 + q * 32;  // first output row of this warp
        if (p.out_f32 || partial) {
          // fp32: stage 16 rows x 32 columns in shared memory (128-byte swizzle) and
          // write them with one TMA store per box: whole 128-byte lines to HBM.  All of
          // this warp's chunks are read before the accumulator is released.
          constexpr bool kTwoSlots = kWarpStore >= 4096;
          uint32_t va[kMine][32];
#pragma unroll
          for (int ci = 0; ci < kMine; ++ci) {
            if (ti.nkb > 0) {
              tmem_ld32(ta + (c0 + ci) * 32, va[ci]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) va[ci][i] = 0;
            }
          }
          if (ti.nkb > 0) {
            tmem_wait_ld();
#pragma unroll
            for (int ci = 0; ci < kMine; ++ci) tmem_tie(va[ci]);
          }
          release();
          // a partial sum always overwrites its slot; the result is added into the output
          // when the call accumulates
          auto put = [&](int ci, int hh, uint8_t* sbuf) {
            if (p.accumulate && !partial)
              tma_reduce_add_2d(tmo, ti.n0 + (c0 + ci) * 32, (int)(orow0 + 16 * hh), sbuf);
            else
              tma_store_2d(tmo, ti.n0 + (c0 + ci) * 32, (int)(orow0 + 16 * hh), sbuf);
          };
          if constexpr (kTwoSlots) {
            // all 32 lanes stage both 16-row boxes of a chunk at once (lane l: row l % 16 of
            // box l / 16, one slot per box), once the previous chunk's stores have read the
            // slots; with half the lanes per box the MMAs beside this epilogue ran ~6 %
            // slower per stage
#pragma unroll
            for (int ci = 0; ci < kMine; ++ci) {
              const uint32_t* v = va[ci];
              if (lane == 0) tma_store_wait_read();
              __syncwarp();
              {
                const int r = lane & 15;
                uint8_t* sbuf = wbuf + (lane >> 4) * 2048;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  *reinterpret_cast<uint4*>(sbuf + r * 128 + ((j ^ (r & 7)) * 16)) =
                      make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                put(ci, 0, wbuf);
                put(ci, 1, wbuf + 2048);
              }
            }
          } else {
            // one 2 KB slot: each box is staged by its 16 lanes after the previous store
            // has read the slot
#pragma unroll
            for (int ci = 0; ci < kMine; ++ci) {
              const uint32_t* v = va[ci];
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                if (lane == 0) tma_store_wait_read();
                __syncwarp();
                if ((lane >> 4) == hh) {
                  const int r = lane & 15;
#pragma unroll
                  for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4*>(wbuf + r * 128 + ((j ^ (r & 7)) * 16)) =
                        make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) put(ci, hh, wbuf);
              }
            }
          }
        } else if (p.accumulate) {
          // bf16 output added to: existing + new in fp32, rounded once, chunk by chunk
          __nv_bfloat16* o = p.out + (orow0 + lane) * p.ld_out + ti.n0 + c0 * 32;
#pragma unroll 1
          for (int ci = 0; ci < kMine; ++ci) {
            uint32_t v[32];
            if (ti.nkb > 0) {
              tmem_ld32(ta + (c0 + ci) * 32, v);
              tmem_wait_ld();
              tmem_tie(v);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = 0;
            }
            const uint4* src = reinterpret_cast<const uint4*>(o + ci * 32);
            uint32_t pk[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const uint4 w = src[q4];
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const int i = 4 * q4 + h;
                pk[i] = pack_bf16(bf_lo(ww[h]) + __uint_as_float(v[2 * i]),
                                  bf_hi(ww[h]) + __uint_as_float(v[2 * i + 1]));
              }
            }
            store_64B(o + ci * 32, pk);
          }
          release();
        } else {
          __nv_bfloat16* o = p.out + (orow0 + lane) * p.ld_out + ti.n0 + c0 * 32;
          uint32_t pk[kMine][16];
#pragma unroll
          for (int ci = 0; ci < kMine; ++ci) {
            if (ti.nkb > 0) {
              uint32_t v[32];
              tmem_ld32(ta + (c0 + ci) * 32, v);
              tmem_wait_ld();
              tmem_tie(v);
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[ci][i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[ci][i] = 0;
            }
          }
          release();
#pragma unroll
          for (int ci = 0; ci < kMine; ++ci) store_64B(o + ci * 32, pk[ci]);
        }
      }
      ++acc_it;
    }
  }
  if constexpr (EPI == EPI_WGRAD || EPI == EPI_STORE || EPI == EPI_SWIGLU_FWD || EPI == EPI_SWIGLU_BWD) {
    if (warp >= 2 && lane == 0) tma_store_wait_all();  // this warp's stores have left shared memory
  }
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the leader's MMAs read the peer's shared memory and TMEM
  if (warp == 0) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Weight gradients of groups cut into K ranges: dW[g] = sum over j (in order) of the fp32
// partial sums in slots (slot prefix of g) + j; groups that were not cut are skipped.
__global__ void __launch_bounds__(256)
wgrad_reduce_kernel(const int32_t* __restrict__ offsets, int kc, int64_t mn4,
                    const float4* __restrict__ part, float4* __restrict__ out32,
                    __nv_bfloat16* __restrict__ out16, int accumulate) {
  __shared__ int s_red[8];
  const int g = blockIdx.y;
  int ns, ck;
  wgrad_split(offsets[g + 1] - offsets[g], kc, ns, ck);
  if (ns <= 1) return;
  int acc = 0;  // partial slots of the groups before g
  for (int e = threadIdx.x; e < g; e += blockDim.x) {
    int n2, c2;
    wgrad_split(offsets[e + 1] - offsets[e], kc, n2, c2);
    acc += n2 > 1 ? n2 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = acc;
  __syncthreads();
  int slot0 = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) slot0 += s_red[w];
  const float4* src = part + (int64_t)slot0 * mn4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < mn4; i += (int64_t)gridDim.x * blockDim.x) {
    float4 a = src[i];
    for (int j = 1; j < ns; ++j) {
      const float4 b = src[(int64_t)j * mn4 + i];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    // the K ranges are summed first; an accumulating call then adds that sum to the output
    if (out32) {
      float4* o = out32 + (int64_t)g * mn4 + i;
      if (accumulate) {
        const float4 b = *o;
        a = make_float4(b.x + a.x, b.y + a.y, b.z + a.z, b.w + a.w);
      }
      *o = a;
    } else {
      uint2* o = reinterpret_cast<uint2*>(out16 + ((int64_t)g * mn4 + i) * 4);
      if (accumulate) {
        const uint2 b = *o;
        a = make_float4(bf_lo(b.x) + a.x, bf_hi(b.x) + a.y, bf_lo(b.y) + a.z, bf_hi(b.y) + a.w);
      }
      uint2 pk;
      pk.x = pack_bf16(a.x, a.y);
      pk.y = pack_bf16(a.z, a.w);
      *o = pk;
    }
  }
}

// ------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

cudaError_t get_encode() {
  if (g_encode) return cudaSuccess;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  cudaError_t err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (err != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

// 2-D tensor map over [outer, inner] with row stride `ld` elements, 128-byte swizzle.
// Elements are bf16, fp32 (f32) or bytes (u8: E4M3 codes).
bool tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
          uint32_t box_inner, uint32_t box_outer, bool f32 = false, bool u8 = false) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {ld * (u8 ? 1 : (f32 ? 4 : 2))};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  const CUtensorMapDataType dt = u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                    : (f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  return g_encode(tm, dt, 2,
                  const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An array of 512-byte scale atoms as a [2 x natoms, 256] byte tensor whose 256 x 2 box is
// one atom (the CTA-pair form of the TMA load then brings it in on the leader's barrier).
bool tmap_atoms(CUtensorMap* tm, const void* base, uint64_t natoms) {
  const cuuint64_t dims[2] = {256, 2 * natoms};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, 2};
  const cuuint32_t es[2] = {1, 1};
  return g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Failure-path test hooks, read once from the environment (unset in normal use):
// MOE_B200_WAIT_NS sets the limit of every bounded wait of the GEMM kernels, and
// MOE_B200_TEST_DROP_STAGE = n makes CTA 0's producer skip its n-th ring stage (no load,
// no arrival), so that the MMA warp's wait for it runs out and the kernel takes its abort
// path: MOE_ERR_TIMEOUT in the status word, then a clean exit.
struct TestHooks {
  uint64_t wait_ns = 0;
  int drop_it = 0;
};
const TestHooks& gemm_test_hooks() {
  static const TestHooks h = [] {
    TestHooks t;
    if (const char* w = getenv("MOE_B200_WAIT_NS")) t.wait_ns = strtoull(w, nullptr, 10);
    if (const char* d = getenv("MOE_B200_TEST_DROP_STAGE")) t.drop_it = atoi(d);
    return t;
  }();
  return h;
}
GemmParams with_hooks(const GemmParams& p) {
  GemmParams q = p;
  q.wait_ns = gemm_test_hooks().wait_ns;
  q.drop_it = gemm_test_hooks().drop_it;
  return q;
}

// Name of a launch in per-launch timing: the expert-FFN GEMMs start with "gemm_", the
// router's tensor-core GEMMs with "router_".
template <int EPI, bool FP8>
constexpr const char* gemm_name() {
  return EPI == EPI_SWIGLU_FWD   ? (FP8 ? "gemm_swiglu_fwd_mx" : "gemm_swiglu_fwd")
         : EPI == EPI_STORE      ? (FP8 ? "gemm_store_mx" : "gemm_store")
         : EPI == EPI_SWIGLU_BWD ? (FP8 ? "gemm_swiglu_bwd_mx" : "gemm_swiglu_bwd")
         : EPI == EPI_WGRAD      ? (FP8 ? "gemm_wgrad_mx" : "gemm_wgrad")
         : EPI == EPI_ROUTER     ? "router_gemm"
                                 : "router_dx_gemm";
}

template <int BN, bool A_MN, bool B_MN, int EPI, bool GROUP_K>
cudaError_t launch(const GemmParams& p, int64_t tile_bound, cudaStream_t st) {
  auto kern = grouped_gemm_sm100<BN, A_MN, B_MN, EPI, GROUP_K>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<BN, false, EPI>::kSmem);
  if (err != cudaSuccess) return err;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tile_bound, num_sms()));
  ProfScope prof(EPI == EPI_WGRAD && !p.offsets ? "router_dw_gemm" : gemm_name<EPI, false>(), st);
  kern<<<grid, kThreads, Cfg<BN, false, EPI>::kSmem, st>>>(with_hooks(p));
  return cudaGetLastError();
}

// MXFP8 variant: 128 x BN tiles of E4M3 operands with E8M0 block scales.
template <int BN, bool A_MN, bool B_MN, int EPI, bool GROUP_K>
cudaError_t launch_mx(const GemmParams& p, int64_t tile_bound, cudaStream_t st) {
  auto kern = grouped_gemm_sm100<BN, A_MN, B_MN, EPI, GROUP_K, false, true>;
  constexpr size_t smem = Cfg<BN, false, EPI, true>::kSmem;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tile_bound, num_sms()));
  ProfScope prof(gemm_name<EPI, true>(), st);
  kern<<<grid, kThreads, smem, st>>>(with_hooks(p));
  return cudaGetLastError();
}

// CTA-pair variant: clusters of 2 CTAs, as many as can be resident at once.
template <int BN, bool B_MN, int EPI, bool FP8 = false, bool GROUP_K = false>
cudaError_t launch_pair(const GemmParams& p, int64_t pair_tile_bound, cudaStream_t st) {
  auto kern = grouped_gemm_sm100<BN, false, B_MN, EPI, GROUP_K, true, FP8>;
  constexpr size_t smem = Cfg<BN, true, EPI, FP8>::kSmem;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_clusters[64] = {0};
  int dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if (dev < 64 && max_clusters[dev] == 0) {
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = num_sms() / 2;
    max_clusters[dev] = n;
  }
  const int clusters = (int)std::max<int64_t>(1, std::min<int64_t>(pair_tile_bound, dev < 64 ? max_clusters[dev] : num_sms() / 2));
  cfg.gridDim = dim3(2 * clusters);
  ProfScope prof(gemm_name<EPI, FP8>(), st);
  return cudaLaunchKernelEx(&cfg, kern, with_hooks(p));
}

// 256-wide MXFP8 tiles where N allows (twice the work per MMA instruction), else 128.
// `units` is the tile count per 128 columns of N.
template <bool A_MN, bool B_MN, int EPI, bool GROUP_K>
cudaError_t launch_mx_n(const GemmParams& p, int N, int64_t units, cudaStream_t st) {
  if (N % 256 == 0) return launch_mx<256, A_MN, B_MN, EPI, GROUP_K>(p, units * (N / 256), st);
  return launch_mx<128, A_MN, B_MN, EPI, GROUP_K>(p, units * (N / 128), st);
}

// K threshold above which a weight-gradient group is cut into several K ranges: one tile
// would carry more than an SM's fair share of the launch's K work (rows x tiles per group /
// SMs), as when most tokens choose one expert; never less than 2048 rows.  (A lower
// threshold was measured: at a quarter of the fair share the partial sums and their
// reduction cost more than the better balance saved on the benchmark workloads.)
int wgrad_kchunk(int64_t rows, int M, int N, int BN) {
  const int64_t per = (int64_t)(M / BM) * (N / BN);
  int64_t kc = (rows * per + num_sms() - 1) / num_sms();
  kc = std::max<int64_t>(kc, 2048);
  return (int)((kc + 127) & ~int64_t(127));
}
// partial slots: a group of c > kc rows takes ceil(c / kc) <= 2 c / kc of them
int64_t wgrad_slots(int64_t rows, int kc) { return 2 * rows / kc + 1; }
int wgrad_bn(int N, bool fp8) { return (!fp8 || N % 256 == 0) ? 256 : 128; }
// MXFP8 weight gradients on CTA pairs (256 x 256 tiles) when M and N are multiples of 256;
// MOE_B200_PAIR=0 turns pairs off here too (read per call: tests switch it)
bool wgrad_pairs(int M, int N) {
  const char* env = getenv("MOE_B200_PAIR");
  if (env && env[0] == '0') return false;
  return M % 256 == 0 && N % 256 == 0;
}

// Sets the split fields of a weight-gradient launch (M x N per group) and returns the
// partial-buffer bytes it may use; `part` may be null when only the size is wanted.
size_t wgrad_setup(GemmParams* p, int64_t rows, int M, int N, bool fp8, float* part) {
  const int kc = wgrad_kchunk(rows, M, N, wgrad_bn(N, fp8));
  const int64_t slots = wgrad_slots(rows, kc);
  if (p) {
    p->kchunk = kc;
    p->part = part;
    if (part && !tmap(&p->tmPart, part, N, (uint64_t)slots * M, N, 32, 16, true)) p->part = nullptr;
  }
  return (size_t)slots * M * N * sizeof(float);
}

cudaError_t wgrad_reduce_launch(const GemmParams& p, int64_t M, int64_t N, float* out32,
                                __nv_bfloat16* out16, cudaStream_t st) {
  const int64_t mn4 = M * N / 4;
  dim3 grid((unsigned)std::min<int64_t>((mn4 + 255) / 256, 16), (unsigned)p.E);
  ProfScope prof("gemm_wgrad_reduce", st);
  wgrad_reduce_kernel<<<grid, 256, 0, st>>>(p.offsets, p.kchunk, mn4, reinterpret_cast<const float4*>(p.part),
                                            reinterpret_cast<float4*>(out32), out16, p.accumulate);
  return cudaGetLastError();
}

GemmParams base_params(const FfnShape& s, const int32_t* offsets, int* status) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.offsets = offsets;
  p.E = s.E;
  p.f = s.f;
  p.status = status;
  return p;
}

int64_t m_tile_bound(const FfnShape& s) { return s.rows / BM + s.E; }
int64_t pair_tile_bound(const FfnShape& s) { return s.rows / (2 * BM) + s.E; }

// CTA pairs (256-row tiles, each weight tile read once per pair) pay off when experts hold
// a few hundred rows or more; with fewer the ragged last tile of every expert wastes more
// (at 512 rows per expert pairs still took 2 % off the step).  MOE_B200_PAIR=0/1 forces
// a mode.
bool use_pairs(const FfnShape& s) {
  const char* env = getenv("MOE_B200_PAIR");  // read per call: tests switch it
  if (env && env[0] == '0') return false;
  if (env && env[0] == '1') return true;
  return s.E > 0 && s.rows / s.E >= 512;
}

template <int BN>
cudaError_t route_tc_bn(const RouteArgs& a, int nb, cudaStream_t st) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  if (!tmap(&p.tmA, a.x, a.d, a.T, a.d, 64, 128) ||
      !tmap(&p.tmB, a.w_router, a.d, a.E, a.d, 64, Cfg<BN, false, EPI_ROUTER>::kBoxRows))
    return cudaErrorInvalidValue;
  p.offsets = nullptr;
  p.E = 1;
  p.rows_total = a.T;
  p.N = a.E;
  p.K = a.d;
  p.topk = a.k;
  p.nb = nb;
  p.bias = a.bias;
  p.logits = a.logits;
  p.topk_idx = a.topk_idx;
  p.topk_gate = a.topk_gate;
  p.blockcounts = a.blockcounts;
  p.localrank = a.localrank;
  p.status = a.status;
  return launch<BN, false, false, EPI_ROUTER, false>(p, nb, st);
}

}  // namespace

bool route_tc_supported(int E, int k, int d) { return E <= 256 && k <= kRouterKMax && d % BK == 0; }

cudaError_t route_tc_launch(const RouteArgs& a, int nb, cudaStream_t st) {
  cudaError_t err = get_encode();
  if (err != cudaSuccess) return err;
  if (a.E <= 16) return route_tc_bn<16>(a, nb, st);
  if (a.E <= 64) return route_tc_bn<64>(a, nb, st);
  if (a.E <= 128) return route_tc_bn<128>(a, nb, st);
  return route_tc_bn<256>(a, nb, st);
}

bool route_bwd_tc_supported(int E, int k, int d) {
  return E % BM == 0 && k <= kRouterKMax && d % 256 == 0;
}

cudaError_t route_bwd_tc_launch(const void* x, const void* w_router, const void* dl_bf16,
                                const void* dx_perm, const int32_t* slot_row, void* dx,
                                float* partial, int splits, int T, int d, int E, int k,
                                int* status, cudaStream_t st) {
  cudaError_t err = get_encode();
  if (err != cudaSuccess) return err;
  // dx = dl W_r + sum_j dx_perm[slot_row[t, j]]   (M = T, N = d, K = E)
  GemmParams p1;
  memset(&p1, 0, sizeof(p1));
  if (!tmap(&p1.tmA, dl_bf16, E, T, E, 64, 128) || !tmap(&p1.tmB, w_router, d, E, d, 64, 64))
    return cudaErrorInvalidValue;
  p1.E = 1; p1.rows_total = T; p1.N = d; p1.K = E; p1.topk = k;
  p1.slot_row = slot_row;
  p1.act = static_cast<const __nv_bfloat16*>(dx_perm); p1.ld_act = d;
  p1.out = static_cast<__nv_bfloat16*>(dx); p1.ld_out = d;
  p1.status = status;
  if ((err = launch<256, false, true, EPI_ROUTER_DX, false>(p1, (int64_t)((T + BM - 1) / BM) * (d / 256), st)) != cudaSuccess)
    return err;
  // partial[s] = dl_s^T x_s over `splits` consecutive token ranges  (M = E, N = d)
  GemmParams p2;
  memset(&p2, 0, sizeof(p2));
  if (!tmap(&p2.tmA, dl_bf16, E, T, E, 64, 64) || !tmap(&p2.tmB, x, d, T, d, 64, 64) ||
      !tmap(&p2.tmOut, partial, d, (uint64_t)splits * E, d, 32, 16, true))
    return cudaErrorInvalidValue;
  p2.E = splits; p2.rows_total = T; p2.split = (T + splits - 1) / splits;
  p2.M = E; p2.N = d;
  p2.out_f32 = partial; p2.ld_out = d; p2.out_group = (int64_t)E * d;
  p2.status = status;
  return launch<256, true, true, EPI_WGRAD, true>(p2, (int64_t)splits * (E / BM) * (d / 256), st);
}

cudaError_t ffn_fwd_bf16(const FfnShape& s, const void* x_perm, const int32_t* offsets,
                         const void* w1, const void* w2, void* act, void* y_perm, int* status,
                         cudaStream_t st) {
  if (s.rows == 0) return cudaSuccess;
  cudaError_t err = get_encode();
  if (err != cudaSuccess) return err;
  const int d = s.d, f = s.f, E = s.E;
  const __nv_bfloat16* actb = static_cast<const __nv_bfloat16*>(act);
  // gate/up GEMM + SwiGLU: act = [a | u | h]
  GemmParams p1 = base_params(s, offsets, status);
  if (!tmap(&p1.tmA, x_perm, d, s.rows, d, 64, 128) ||
      !tmap(&p1.tmB, w1, d, (uint64_t)E * 2 * f, d, 64, 128))
    return cudaErrorInvalidValue;
  p1.N = f; p1.K = d; p1.b_rows = 2 * f;
  p1.out = static_cast<__nv_bfloat16*>(act); p1.ld_out = 3 * f;
  if (!tmap(&p1.tmOut, act, 3 * f, s.rows, 3 * f, 64, 16)) return cudaErrorInvalidValue;
  const bool pairs = use_pairs(s);
  err = pairs ? launch_pair<256, false, EPI_SWIGLU_FWD>(p1, pair_tile_bound(s) * (f / 128), st)
              : launch<256, false, false, EPI_SWIGLU_FWD, false>(p1, m_tile_bound(s) * (f / 128), st);
  if (err != cudaSuccess) return err;
  if (!y_perm) return cudaSuccess;  // recompute of a | u | h only
  // down GEMM: y = h W2^T
  GemmParams p2 = base_params(s, offsets, status);
  if (!tmap(&p2.tmA, actb + 2 * f, f, s.rows, 3 * f, 64, 128) ||
      !tmap(&p2.tmB, w2, f, (uint64_t)E * d, f, 64, 128))
    return cudaErrorInvalidValue;
  p2.N = d; p2.K = f; p2.b_rows = d;
  p2.out = static_cast<__nv_bfloat16*>(y_perm); p2.ld_out = d;
  if (!tmap(&p2.tmOut, y_perm, d, s.rows, d, 64, 16)) return cudaErrorInvalidValue;
  return pairs ? launch_pair<256, false, EPI_STORE>(p2, pair_tile_bound(s) * (d / 256), st)
               : launch<256, false, false, EPI_STORE, false>(p2, m_tile_bound(s) * (d / 256), st);
}

cudaError_t ffn_bwd_bf16(const FfnShape& s, const void* dy_perm, const void* x_perm,
                         const void* act, const int32_t* offsets, const void* w1, const void* w2,
                         void* dx_perm, void* dw1, void* dw2, bool dw_f32, void* scratch,
                         int* status, cudaStream_t st,
                         bool accumulate) {
  cudaError_t err = get_encode();
  if (err != cudaSuccess) return err;
  const int d = s.d, f = s.f, E = s.E;
  const __nv_bfloat16* actb = static_cast<const __nv_bfloat16*>(act);
  __nv_bfloat16* dadu = static_cast<__nv_bfloat16*>(scratch);
  const uint64_t rows_tm = std::max<int64_t>(s.rows, 1);  // tensor maps need a non-zero extent
  if (s.rows > 0) {
    // dgrad 1: dh = dy W2[e], fused SwiGLU backward -> dadu = [da | du]
    GemmParams p3 = base_params(s, offsets, status);
    if (!tmap(&p3.tmA, dy_perm, d, s.rows, d, 64, 128) ||
        !tmap(&p3.tmB, w2, f, (uint64_t)E * d, f, 64, 64))
      return cudaErrorInvalidValue;
    p3.N = f; p3.K = d; p3.b_rows = d;
    p3.out = dadu; p3.ld_out = 2 * f;
    if (!tmap(&p3.tmOut, dadu, 2 * f, s.rows, 2 * f, 64, 16)) return cudaErrorInvalidValue;
    p3.act = actb; p3.ld_act = 3 * f;
    if (reinterpret_cast<uintptr_t>(actb) & 31) return cudaErrorInvalidValue;  // 32-byte a/u loads
    const bool pairs = use_pairs(s);
    err = pairs ? launch_pair<256, true, EPI_SWIGLU_BWD>(p3, pair_tile_bound(s) * (f / 256), st)
                : launch<256, false, true, EPI_SWIGLU_BWD, false>(p3, m_tile_bound(s) * (f / 256), st);
    if (err != cudaSuccess) return err;
    // dgrad 2: dx = [da | du] W1[e]
    GemmParams p4 = base_params(s, offsets, status);
    if (!tmap(&p4.tmA, dadu, 2 * f, s.rows, 2 * f, 64, 128) ||
        !tmap(&p4.tmB, w1, d, (uint64_t)E * 2 * f, d, 64, 64))
      return cudaErrorInvalidValue;
    p4.N = d; p4.K = 2 * f; p4.b_rows = 2 * f;
    p4.out = static_cast<__nv_bfloat16*>(dx_perm); p4.ld_out = d;
    if (!tmap(&p4.tmOut, dx_perm, d, s.rows, d, 64, 16)) return cudaErrorInvalidValue;
    err = pairs ? launch_pair<256, true, EPI_STORE>(p4, pair_tile_bound(s) * (d / 256), st)
                : launch<256, false, true, EPI_STORE, false>(p4, m_tile_bound(s) * (d / 256), st);
    if (err != cudaSuccess) return err;
  }
  // wgrad 2: dW2[e] = dy^T h   (M = d, N = f, K = the expert's rows)
  GemmParams p5 = base_params(s, offsets, status);
  if (!tmap(&p5.tmA, dy_perm, d, rows_tm, d, 64, 64) ||
      !tmap(&p5.tmB, actb + 2 * f, f, rows_tm, 3 * f, 64, 64))
    return cudaErrorInvalidValue;
  p5.M = d; p5.N = f;
  p5.out = static_cast<__nv_bfloat16*>(dw2); p5.out_f32 = dw_f32 ? static_cast<float*>(dw2) : nullptr;
  p5.ld_out = f; p5.out_group = (int64_t)d * f; p5.accumulate = accumulate;
  if (dw_f32 && !tmap(&p5.tmOut, dw2, f, (uint64_t)E * d, f, 32, 16, true)) return cudaErrorInvalidValue;
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(scratch) +
                                         align256((size_t)s.rows * 2 * f * 2));
  wgrad_setup(&p5, s.rows, d, f, false, part);
  if (!p5.part) return cudaErrorInvalidValue;
  if ((err = launch<256, true, true, EPI_WGRAD, true>(p5, num_sms(), st)) != cudaSuccess ||
      (err = wgrad_reduce_launch(p5, d, f, p5.out_f32, p5.out, st)) != cudaSuccess)
    return err;
  // wgrad 1: dW1[e] = [da | du]^T x   (M = 2f, N = d)
  GemmParams p6 = base_params(s, offsets, status);
  if (!tmap(&p6.tmA, dadu, 2 * f, rows_tm, 2 * f, 64, 64) ||
      !tmap(&p6.tmB, x_perm, d, rows_tm, d, 64, 64))
    return cudaErrorInvalidValue;
  p6.M = 2 * f; p6.N = d;
  p6.out = static_cast<__nv_bfloat16*>(dw1); p6.out_f32 = dw_f32 ? static_cast<float*>(dw1) : nullptr;
  p6.ld_out = d; p6.out_group = (int64_t)2 * f * d; p6.accumulate = accumulate;
  if (dw_f32 && !tmap(&p6.tmOut, dw1, d, (uint64_t)E * 2 * f, d, 32, 16, true)) return cudaErrorInvalidValue;
  wgrad_setup(&p6, s.rows, 2 * f, d, false, part);
  if (!p6.part) return cudaErrorInvalidValue;
  if ((err = launch<256, true, true, EPI_WGRAD, true>(p6, num_sms(), st)) != cudaSuccess) return err;
  return wgrad_reduce_launch(p6, 2 * f, d, p6.out_f32, p6.out, st);
}

size_t wgrad_part_bytes(const FfnShape& s, bool fp8) {
  return std::max(wgrad_setup(nullptr, s.rows, s.d, s.f, fp8, nullptr),
                  wgrad_setup(nullptr, s.rows, 2 * s.f, s.d, fp8, nullptr));
}


// ---------------------------------------------------------------- MXFP8 FFN
// Activations arrive and leave in bf16; each GEMM operand is quantised along that
// GEMM's K right before it is used (forward: x and h along their rows; dgrad: dy and
// [da|du] along their rows, the weights along their rows of K via the moe_mx_weights
// copies; wgrad: dy, h, [da|du] and x in 32-row blocks that restart at every expert's
// first row).  Accumulation is fp32; outputs are bf16 (dW fp32).  Scales are kept as
// the MMA's 512-byte atoms in the order the GEMM reads them (see mxfp8.cu).
namespace {

struct MxLayout {
  // kept from the forward to the backward: the token-block copies of x and h
  size_t qx1, sx1, qh1, sh1;
  size_t rt, map, cnt;                                // row -> tile map, token-block map
  size_t qx0, sx0, qh0, sh0;                          // forward row copies
  size_t dadu, qdy0, sdy0, qda0, sda0;                // backward, dgrad operands
  size_t qdy1, sdy1, qda1, sda1;                      // backward, wgrad operands
  size_t part;                                        // split weight-gradient partial sums
  size_t fwd_bytes, bwd_bytes;
};

MxLayout mx_layout(const FfnShape& s) {
  const size_t R = (size_t)s.rows, d = s.d, f = s.f;
  // at most R/128 + E tiles (row-grouped) or stages (segmented) of 128 rows; an atom
  // covers 128 rows x 128 K elements
  const size_t tiles = R / 128 + s.E;
  auto atoms = [&](size_t K) { return tiles * (K / 128) * 512; };
  // token-block copies: [K][Rp], the token axis padded to whole 128-row stages per expert
  const size_t Rp = tiles * 128;
  MxLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o += align256(bytes); return at; };
  L.qx1 = take(Rp * d); L.sx1 = take(atoms(d));
  L.qh1 = take(Rp * f); L.sh1 = take(atoms(f));
  L.rt = take(R * 4);
  L.map = take((R / 32 + s.E) * 16 + (R / 128 + s.E + 1) * 4);  // block map, stage table
  L.cnt = take(8);
  const size_t base = o;
  L.qx0 = take(R * d); L.sx0 = take(atoms(d)); L.qh0 = take(R * f); L.sh0 = take(atoms(f));
  L.fwd_bytes = o;
  o = base;
  L.dadu = take(R * 2 * f * 2);
  L.qdy0 = take(R * d); L.sdy0 = take(atoms(d));
  L.qda0 = take(R * 2 * f); L.sda0 = take(atoms(2 * f));
  L.qdy1 = take(Rp * d); L.sdy1 = take(atoms(d));
  L.qda1 = take(Rp * 2 * f); L.sda1 = take(atoms(2 * f));
  L.part = take(wgrad_part_bytes(s, true));
  L.bwd_bytes = o;
  return L;
}

GemmParams mx_params(const FfnShape& s, const int32_t* offsets, int* status) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.offsets = offsets;
  p.E = s.E;
  p.f = s.f;
  p.status = status;
  p.rows_total = (int)s.rows;
  return p;
}

}  // namespace

size_t ffn_mx_ws_bytes(const FfnShape& s) {
  const MxLayout L = mx_layout(s);
  return std::max(L.fwd_bytes, L.bwd_bytes);
}

void ffn_mx_ws_regions(const FfnShape& s, size_t out[kMxRegions]) {
  const MxLayout L = mx_layout(s);
  const size_t r[kMxRegions] = {L.qx1, L.sx1, L.qh1, L.sh1, L.rt, L.map, L.cnt,
                                L.qx0, L.sx0, L.qh0, L.sh0, L.dadu, L.qdy0, L.sdy0,
                                L.qda0, L.sda0, L.qdy1, L.sdy1, L.qda1, L.sda1};
  for (int i = 0; i < kMxRegions; ++i) out[i] = r[i];
}

cudaError_t mx_quantize_weights(int E, int d, int f, const float* w1, const float* w2,
                                const MxWeights& w, cudaStream_t st) {
  auto u8 = [](const uint8_t* p) { return const_cast<uint8_t*>(p); };
  cudaError_t err = mxfp8_weights(w1, E, 2 * f, d, u8(w.w1_q), u8(w.w1_s), u8(w.w1t_q),
                                  u8(w.w1t_s), st);
  if (err != cudaSuccess) return err;
  return mxfp8_weights(w2, E, d, f, u8(w.w2_q), u8(w.w2_s), u8(w.w2t_q), u8(w.w2t_s), st);
}

cudaError_t ffn_fwd_mx(const FfnShape& s, const void* x_perm, const int32_t* offsets,
                       const MxWeights& w, void* act, void* y_perm, void* scratch, int* status,
                       cudaStream_t st) {
  if (s.rows == 0) return cudaSuccess;
  cudaError_t err = get_encode();
  if (err != cudaSuccess) return err;
  const int d = s.d, f = s.f, E = s.E;
  const int64_t R = s.rows;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  const MxLayout L = mx_layout(s);
  const __nv_bfloat16* actb = static_cast<const __nv_bfloat16*>(act);
  int32_t* rt = reinterpret_cast<int32_t*>(ws + L.rt);
  int4* map = reinterpret_cast<int4*>(ws + L.map);
  int32_t* smap = reinterpret_cast<int32_t*>(ws + L.map + (s.rows / 32 + s.E) * 16);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  // x along d (gate/up GEMM) and in token blocks (kept for the dW1 GEMM of the backward);
  // without x_perm, the fused dispatch has written both copies and the maps already
  if (x_perm) {
    if ((err = row_tile_launch(offsets, E, R, rt, st)) != cudaSuccess ||
        (err = seg_blocks_launch(offsets, E, map, cnt, smap, st)) != cudaSuccess ||
        (err = mxfp8_act(R, E, d, d, x_perm, map, cnt, smap, rt, ws + L.qx0, ws + L.sx0, ws + L.qx1,
                         ws + L.sx1, st)) != cudaSuccess)
      return err;
  }
  GemmParams p1 = mx_params(s, offsets, status);
  if (!tmap(&p1.tmA, ws + L.qx0, d, R, d, 128, 128, false, true) ||
      !tmap(&p1.tmB, w.w1_q, d, (uint64_t)E * 2 * f, d, 128, 128, false, true) ||
      !tmap(&p1.tmOut, act, 3 * f, R, 3 * f, 64, 16))
    return cudaErrorInvalidValue;
  p1.sfa = ws + L.sx0;
  p1.sfb = w.w1_s;
  p1.N = f; p1.K = d; p1.b_rows = 2 * f;
  p1.out = static_cast<__nv_bfloat16*>(act); p1.ld_out = 3 * f;
  // h's two MXFP8 copies come from the gate/up epilogue (MOE_B200_HMX=0: from a pass of
  // the activation quantiser over the bf16 h instead; read per call, tests compare them)
  const char* hmx_env = getenv("MOE_B200_HMX");
  const bool h_mx = !(hmx_env && hmx_env[0] == '0');
  if (h_mx) {
    p1.mx_q_r = ws + L.qh0;
    p1.mx_s_r = ws + L.sh0;
    p1.mx_q_c = ws + L.qh1;
    p1.mx_s_c = ws + L.sh1;
    p1.mx_rp = ((int64_t)R / 128 + E) * 128;
  }
  // 128 gate + 128 up columns per tile; CTA pairs where experts are large enough
  const bool pairs = use_pairs(s);
  const uint64_t tiles = (uint64_t)R / 128 + E;  // row-tile atoms per 128 columns of K
  if (pairs) {
    if (!tmap_atoms(&p1.tmSfa, ws + L.sx0, tiles * (d / 128)) ||
        !tmap_atoms(&p1.tmSfb, w.w1_s, (uint64_t)E * 2 * f * d / (32 * 512)))
      return cudaErrorInvalidValue;
    err = launch_pair<256, false, EPI_SWIGLU_FWD, true>(p1, pair_tile_bound(s) * (f / 128), st);
  } else {
    err = launch_mx<256, false, false, EPI_SWIGLU_FWD, false>(p1, m_tile_bound(s) * (f / 128), st);
  }
  if (err != cudaSuccess) return err;
  // h along f (down GEMM) and in token blocks (kept for the dW2 GEMM of the backward)
  if (!h_mx &&
      (err = mxfp8_act(R, E, f, 3 * f, actb + 2 * f, map, cnt, smap, rt, ws + L.qh0, ws + L.sh0,
                       ws + L.qh1, ws + L.sh1, st)) != cudaSuccess)
    return err;
  if (!y_perm) return cudaSuccess;  // recompute: a | u | h and the token-block copies only
  GemmParams p2 = mx_params(s, offsets, status);
  if (!tmap(&p2.tmA, ws + L.qh0, f, R, f, 128, 128, false, true) ||
      !tmap(&p2.tmB, w.w2_q, f, (uint64_t)E * d, f, 128, 128, false, true) ||
      !tmap(&p2.tmOut, y_perm, d, R, d, 64, 16))
    return cudaErrorInvalidValue;
  p2.sfa = ws + L.sh0;
  p2.sfb = w.w2_s;
  p2.N = d; p2.K = f; p2.b_rows = d;
  p2.out = static_cast<__nv_bfloat16*>(y_perm); p2.ld_out = d;
  if (pairs && d % 256 == 0) {
    if (!tmap_atoms(&p2.tmSfa, ws + L.sh0, tiles * (f / 128)) ||
        !tmap_atoms(&p2.tmSfb, w.w2_s, (uint64_t)E * d * f / (32 * 512)))
      return cudaErrorInvalidValue;
    return launch_pair<256, false, EPI_STORE, true>(p2, pair_tile_bound(s) * (d / 256), st);
  }
  return launch_mx_n<false, false, EPI_STORE, false>(p2, d, m_tile_bound(s), st);
}

cudaError_t mx_dispatch(const FfnShape& s, const void* x, const int32_t* perm_src,
                        const int32_t* offsets, void* scratch, cudaStream_t st) {
  if (s.rows == 0) return cudaSuccess;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  const MxLayout L = mx_layout(s);
  int32_t* rt = reinterpret_cast<int32_t*>(ws + L.rt);
  int4* map = reinterpret_cast<int4*>(ws + L.map);
  int32_t* smap = reinterpret_cast<int32_t*>(ws + L.map + (s.rows / 32 + s.E) * 16);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  cudaError_t err;
  if ((err = row_tile_launch(offsets, s.E, s.rows, rt, st)) != cudaSuccess ||
      (err = seg_blocks_launch(offsets, s.E, map, cnt, smap, st)) != cudaSuccess)
    return err;
  return mxfp8_act(s.rows, s.E, s.d, s.d, x, map, cnt, smap, rt, ws + L.qx0, ws + L.sx0, ws + L.qx1,
                   ws + L.sx1, st, perm_src);
}

cudaError_t mx_combine_bwd(const FfnShape& s, const void* dout, const void* y_perm,
                           const int32_t* slot_row, const float* gate, const int32_t* perm_src,
                           float* dgate, int T, int k, void* scratch, cudaStream_t st) {
  cudaError_t err = combine_bwd_launch(true, dout, y_perm, slot_row, gate, nullptr, dgate, T, s.d,
                                       k, st);
  if (err != cudaSuccess || s.rows == 0) return err;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  const MxLayout L = mx_layout(s);
  int32_t* rt = reinterpret_cast<int32_t*>(ws + L.rt);
  int4* map = reinterpret_cast<int4*>(ws + L.map);
  int32_t* smap = reinterpret_cast<int32_t*>(ws + L.map + (s.rows / 32 + s.E) * 16);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  // each routed row's gate, in the permuted order, where [da | du] goes later
  float* gate_perm = reinterpret_cast<float*>(ws + L.dadu);
  if ((err = perm_gate_launch(slot_row, gate, gate_perm, T, k, st)) != cudaSuccess) return err;
  return mxfp8_act(s.rows, s.E, s.d, s.d, dout, map, cnt, smap, rt, ws + L.qdy0, ws + L.sdy0,
                   ws + L.qdy1, ws + L.sdy1, st, perm_src, gate_perm);
}

cudaError_t ffn_bwd_mx(const FfnShape& s, const void* dy_perm, const void* x_perm, const void* act,
                       const int32_t* offsets, const MxWeights& w, void* dx_perm, float* dw1,
                       float* dw2, void* scratch, int* status, cudaStream_t st,
                       bool accumulate) {
  cudaError_t err = get_encode();
  if (err != cudaSuccess) return err;
  const int d = s.d, f = s.f, E = s.E;
  const int64_t R = s.rows;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  const MxLayout L = mx_layout(s);
  const __nv_bfloat16* actb = static_cast<const __nv_bfloat16*>(act);
  __nv_bfloat16* dadu = reinterpret_cast<__nv_bfloat16*>(ws + L.dadu);
  int32_t* rt = reinterpret_cast<int32_t*>(ws + L.rt);
  int4* map = reinterpret_cast<int4*>(ws + L.map);
  int32_t* smap = reinterpret_cast<int32_t*>(ws + L.map + (s.rows / 32 + s.E) * 16);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  (void)x_perm;  // its token-block copy comes from the forward
  if (R > 0) {
    // (the row-tile and token-block maps of the forward are still in the workspace)
    // dgrad 1: dh = dy W2 (dy along d, W2 along its d rows), SwiGLU backward -> [da | du];
    // dy also in token blocks for the dW2 GEMM
    // (without dy_perm, the fused combine backward has written both copies already)
    if (dy_perm &&
        (err = mxfp8_act(R, E, d, d, dy_perm, map, cnt, smap, rt, ws + L.qdy0, ws + L.sdy0, ws + L.qdy1,
                         ws + L.sdy1, st)) != cudaSuccess)
      return err;
    GemmParams p3 = mx_params(s, offsets, status);
    if (!tmap(&p3.tmA, ws + L.qdy0, d, R, d, 128, 128, false, true) ||
        !tmap(&p3.tmB, w.w2t_q, f, (uint64_t)E * d, f, 128, 128, false, true) ||
        !tmap(&p3.tmOut, dadu, 2 * f, R, 2 * f, 64, 16))
      return cudaErrorInvalidValue;
    p3.sfa = ws + L.sdy0;
    p3.sfb = w.w2t_s;
    p3.N = f; p3.K = d; p3.b_rows = d;
    p3.out = dadu; p3.ld_out = 2 * f;
    p3.act = actb; p3.ld_act = 3 * f;
    if (reinterpret_cast<uintptr_t>(actb) & 31) return cudaErrorInvalidValue;  // 32-byte a/u loads
    // [da | du] leaves the SwiGLU-backward epilogue as its two MXFP8 copies (no bf16 round
    // trip); MOE_B200_DADU=0 writes bf16 [da | du] and quantises it in a pass of its own,
    // =keep writes both (read per call: tests compare the forms)
    const char* dadu_env = getenv("MOE_B200_DADU");
    const bool dadu_mx = !(dadu_env && dadu_env[0] == '0');
    if (dadu_mx) {
      p3.mx_q_r = ws + L.qda0;
      p3.mx_s_r = ws + L.sda0;
      p3.mx_q_c = ws + L.qda1;
      p3.mx_s_c = ws + L.sda1;
      p3.mx_rp = ((int64_t)R / 128 + E) * 128;
      if (!(dadu_env && dadu_env[0] == 'k')) p3.out = nullptr;
    }
    const bool pairs = use_pairs(s);
    const uint64_t tiles = (uint64_t)R / 128 + E;
    if (pairs && f % 256 == 0) {
      if (!tmap_atoms(&p3.tmSfa, ws + L.sdy0, tiles * (d / 128)) ||
          !tmap_atoms(&p3.tmSfb, w.w2t_s, (uint64_t)E * d * f / (32 * 512)))
        return cudaErrorInvalidValue;
      err = launch_pair<256, true, EPI_SWIGLU_BWD, true>(p3, pair_tile_bound(s) * (f / 256), st);
    } else {
      err = launch_mx_n<false, true, EPI_SWIGLU_BWD, false>(p3, f, m_tile_bound(s), st);
    }
    if (err != cudaSuccess) return err;
    // dgrad 2: dx = [da | du] W1 ([da | du] along 2f, W1 along its 2f rows); [da | du]
    // also in token blocks for the dW1 GEMM
    if (!dadu_mx &&
        (err = mxfp8_act(R, E, 2 * f, 2 * f, dadu, map, cnt, smap, rt, ws + L.qda0, ws + L.sda0,
                         ws + L.qda1, ws + L.sda1, st)) != cudaSuccess)
      return err;
    GemmParams p4 = mx_params(s, offsets, status);
    if (!tmap(&p4.tmA, ws + L.qda0, 2 * f, R, 2 * f, 128, 128, false, true) ||
        !tmap(&p4.tmB, w.w1t_q, d, (uint64_t)E * 2 * f, d, 128, 128, false, true) ||
        !tmap(&p4.tmOut, dx_perm, d, R, d, 64, 16))
      return cudaErrorInvalidValue;
    p4.sfa = ws + L.sda0;
    p4.sfb = w.w1t_s;
    p4.N = d; p4.K = 2 * f; p4.b_rows = 2 * f;
    p4.out = static_cast<__nv_bfloat16*>(dx_perm); p4.ld_out = d;
    if (pairs && d % 256 == 0) {
      if (!tmap_atoms(&p4.tmSfa, ws + L.sda0, tiles * (2 * f / 128)) ||
          !tmap_atoms(&p4.tmSfb, w.w1t_s, (uint64_t)E * 2 * f * d / (32 * 512)))
        return cudaErrorInvalidValue;
      err = launch_pair<256, true, EPI_STORE, true>(p4, pair_tile_bound(s) * (d / 256), st);
    } else {
      err = launch_mx_n<false, true, EPI_STORE, false>(p4, d, m_tile_bound(s), st);
    }
    if (err != cudaSuccess) return err;
  }
  // wgrad 2: dW2[e] = dy^T h  (M = d, N = f); both operands K-major over the padded
  // token axis ([columns][Rp] token-block copies).  256 x 256 tiles on CTA pairs where
  // M and N allow: each CTA reads half of the B rows, so a tile's operand bytes per MMA
  // fall by a third and the smaller stages leave room for a deeper ring.
  const uint64_t Rp = ((uint64_t)R / 128 + E) * 128;
  const uint64_t stages = (uint64_t)R / 128 + E;  // atoms per 128 columns of a token-block copy
  auto wgrad_mx = [&](GemmParams& pw, const uint8_t* sfa, const uint8_t* sfb, int M, int N) {
    if (wgrad_pairs(M, N)) {
      if (!tmap_atoms(&pw.tmSfa, sfa, stages * (M / 128)) ||
          !tmap_atoms(&pw.tmSfb, sfb, stages * (N / 128)))
        return cudaErrorInvalidValue;
      return launch_pair<256, false, EPI_WGRAD, true, true>(pw, num_sms() / 2, st);
    }
    return launch_mx_n<false, false, EPI_WGRAD, true>(pw, N, num_sms(), st);
  };
  GemmParams p5 = mx_params(s, offsets, status);
  if (!tmap(&p5.tmA, ws + L.qdy1, Rp, d, Rp, 128, 128, false, true) ||
      !tmap(&p5.tmB, ws + L.qh1, Rp, f, Rp, 128, 128, false, true) ||
      !tmap(&p5.tmOut, dw2, f, (uint64_t)E * d, f, 32, 16, true))
    return cudaErrorInvalidValue;
  p5.sfa = ws + L.sdy1;
  p5.sfb = ws + L.sh1;
  p5.M = d; p5.N = f;
  p5.out_f32 = dw2; p5.ld_out = f; p5.out_group = (int64_t)d * f; p5.accumulate = accumulate;
  wgrad_setup(&p5, R, d, f, true, reinterpret_cast<float*>(ws + L.part));
  if (!p5.part) return cudaErrorInvalidValue;
  if ((err = wgrad_mx(p5, ws + L.sdy1, ws + L.sh1, d, f)) != cudaSuccess ||
      (err = wgrad_reduce_launch(p5, d, f, dw2, nullptr, st)) != cudaSuccess)
    return err;
  // wgrad 1: dW1[e] = [da | du]^T x  (M = 2f, N = d)
  GemmParams p6 = mx_params(s, offsets, status);
  if (!tmap(&p6.tmA, ws + L.qda1, Rp, 2 * f, Rp, 128, 128, false, true) ||
      !tmap(&p6.tmB, ws + L.qx1, Rp, d, Rp, 128, 128, false, true) ||
      !tmap(&p6.tmOut, dw1, d, (uint64_t)E * 2 * f, d, 32, 16, true))
    return cudaErrorInvalidValue;
  p6.sfa = ws + L.sda1;
  p6.sfb = ws + L.sx1;
  p6.M = 2 * f; p6.N = d;
  p6.out_f32 = dw1; p6.ld_out = d; p6.out_group = (int64_t)2 * f * d; p6.accumulate = accumulate;
  wgrad_setup(&p6, R, 2 * f, d, true, reinterpret_cast<float*>(ws + L.part));
  if (!p6.part) return cudaErrorInvalidValue;
  if ((err = wgrad_mx(p6, ws + L.sda1, ws + L.sx1, 2 * f, d)) != cudaSuccess) return err;
  return wgrad_reduce_launch(p6, 2 * f, d, dw1, nullptr, st);
}

}  // namespace moe
