// verify_attn.cu — tree-verify MLA-absorb attention on sm_100a tensor cores.
//
// What it computes (sources: "Race Conditions, Buffer Aliasing, and the
// Architecture of a Native DDTree Inference Engine", sections "The Mission: A
// Native DDTree Engine" and "The Cache Compaction Problem"; "The Microsecond
// Verdict: Validating a DDTree Kernel Fix Under Time Pressure", section "The
// Timeout That Tells a Story"): for request b with prefix P and tree block at
// cache rows P .. P+Q-1, every (node i, head h) row attends over the cache rows
// j < P+Q that it may see (all prefix rows; tree row P+a iff a is i or an
// ancestor of i) with score scale * ([q_lat|q_rope] . [c_kv|k_rope]) and value
// c_kv.  The pages' kernel re-read the shared latent cache once per head; here
// each KV tile is fetched once per pair of CTAs and feeds all 128 query rows
// (two tree nodes x 64 heads) they hold.
//
// Design (one CTA pair = one thread-block cluster of 2 on two SMs):
//   * 128 query rows per pair, 64 per CTA (one tree node, all 64 heads), as the
//     M dimension of cta_group::2 tcgen05 MMAs (M = 128).  The accumulator
//     layout of that shape gives each CTA its 64 rows spread over all 128 TMEM
//     lanes: lanes 0-63 hold columns [0, N/2) and lanes 64-127 columns [N/2, N).
//   * S = Q K^T per 128-key tile: 36 MMAs of N = 128, K = 16 (576 = 9 chunks of
//     64).  Q (64 rows x 576, 72 KB per CTA) stays in shared memory; each CTA
//     stages its half of the keys, two 64-dim chunks per ring stage (64 keys x
//     128 dims = 16 KB, one commit per 8 MMAs).
//   * O += P V per tile: 16 MMAs of N = 256, K = 16 into two fp32 accumulators
//     covering the 512 latent columns (128 TMEM columns each per CTA).  V is the
//     same c_kv rows read as an MN-major operand (each CTA stages 128 latent
//     columns x 64 keys = 16 KB per stage, one commit per 4 MMAs).
//   * TMEM per CTA: four S buffers (4 x 64 cols) + O (256 cols) = all 512
//     columns; four S buffers let S = Q K^T run up to three tiles ahead of the
//     softmax.
//   * Built with DDT_VERIFY_TILE_KEYS=256 the tiles hold 256 keys: S = Q K^T
//     runs at N = 256 into two S buffers of 128 columns, each softmax thread
//     takes its 128 keys in two 64-key chunks, and P is 32 KB per buffer.  That
//     build is correct but slower (its shared memory leaves thinner rings), so
//     128-key tiles are the default.
//   * Warp roles: warps 0-3 softmax and epilogue (thread t owns TMEM lane t, i.e.
//     half of one query row); warps 4 and 8 TMA producers of the K rings of
//     even and odd tiles, warp 6 the producer of the V ring; warps 5 and 10
//     issue S = Q K^T for even and odd tiles and warp 7 issues O += P V (the
//     even CTA of the pair issues for both); warp 9 idles.  Three issuing
//     threads keep the tensor core fed while each waits on barriers or commits
//     stages, and they sit on three different SM sub-partitions.
//   * Online softmax in registers with exp2; the row maximum of the two half
//     rows is exchanged through shared memory; O is rescaled lazily, only when
//     the running maximum grows by more than 2^8.
//   * Long caches: the KV tiles of a request are split into num_splits ranges
//     handled by different pairs; each writes a normalised partial output and
//     its log-sum-exp, and a merge kernel combines them.
//   * Cache rows at or past P+Q (padding, possibly non-finite) are never
//     loaded: the last KV tile of a request ends exactly at row P+Q.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "ddt.h"
#include "ddt_internal.h"

namespace ddt {
__device__ unsigned int ddt_fault_word = 0;  // bit set, see ddt_fault_flags
}  // namespace ddt

#include "sm100_ptx.cuh"

namespace ddt {

namespace va {
// S = Q K^T issuers: tile G goes to issuer G % kQKIss, each with its own K ring
// and its own K producer warp.
constexpr int kQKIss = 2;
// Warp roles.  Warp w runs on sub-partition w % 4, and each sub-partition runs
// one softmax warp (warps 0-3: TMEM lane quarter w).  The three threads that
// issue MMAs sit on three different sub-partitions, so no two of them share a
// scheduler: with both S issuers on one sub-partition the kernel ran 3-10 %
// slower.  DDT_VERIFY_WARP_MAP 11 (default): 4 K producer 0 (and Q), 5 S issuer
// 0, 6 V producer, 7 P V issuer, 8 K producer 1, 9 idle, 10 S issuer 1.
// DDT_VERIFY_WARP_MAP 10: the same without the idle warp (6 S issuer 1, 9 V
// producer).
#ifndef DDT_VERIFY_WARP_MAP
#define DDT_VERIFY_WARP_MAP 11
#endif
static_assert(DDT_VERIFY_WARP_MAP == 10 || DDT_VERIFY_WARP_MAP == 11, "warp map 10 or 11");
constexpr int kWarpKProd0 = 4, kWarpSIss0 = 5, kWarpPVIss = 7, kWarpKProd1 = 8;
constexpr int kWarpVProd = DDT_VERIFY_WARP_MAP == 11 ? 6 : 9;
constexpr int kWarpSIss1 = DDT_VERIFY_WARP_MAP == 11 ? 10 : 6;
constexpr int kWarpTmem = kWarpSIss0;  // allocates and frees the tensor memory
constexpr int kThreads = 32 * DDT_VERIFY_WARP_MAP;
constexpr int kSoftmaxThreads = 128;
constexpr int kStageBytes = 8192;                  // Q chunk, P chunk, output box: 64 x 128 B
// KV tile: kTK cache rows per tile; each CTA of the pair stages kKH of them for
// S = Q K^T (the pair's MMA has N = kTK).
constexpr int kTK = DDT_VERIFY_TILE_KEYS;
static_assert(kTK == 128 || kTK == 256, "KV tiles of 128 or 256 rows");
constexpr int kKH = kTK / 2;
// K stage: kKStageChunks 64-dim chunks of kKH keys, committed as one unit after
// their 4 * kKStageChunks MMAs; a tile's 9 chunks (8 latent + 1 rope) fill
// kKStagesPerTile stages, the last one partly when the stages hold two chunks.
// Fewer, larger stages mean fewer commits and barrier round trips per tile: with
// 128-key tiles, two-chunk K stages and 64-key V stages (the defaults) run the
// 64 x 33 x 4096 workload 6 % faster than one-chunk K and 32-key V stages over
// the same ring bytes.
#ifndef DDT_VERIFY_K_STAGE_CHUNKS
#define DDT_VERIFY_K_STAGE_CHUNKS (DDT_VERIFY_TILE_KEYS == 128 ? 2 : 1)
#endif
constexpr int kKStageChunks = DDT_VERIFY_K_STAGE_CHUNKS;
static_assert(kKStageChunks == 1 || kKStageChunks == 2, "K stages of one or two chunks");
constexpr int kKChunkBytes = kKH * 128;            // kKH keys x 64 dims
constexpr int kKStageBytes = kKChunkBytes * kKStageChunks;
#ifndef DDT_VERIFY_K_STAGES
#define DDT_VERIFY_K_STAGES (DDT_VERIFY_TILE_KEYS == 128 && DDT_VERIFY_K_STAGE_CHUNKS == 1 ? 4 : 2)
#endif
#ifndef DDT_VERIFY_V_KEYS
#define DDT_VERIFY_V_KEYS 64
#endif
#ifndef DDT_VERIFY_V_STAGES
#define DDT_VERIFY_V_STAGES (DDT_VERIFY_V_KEYS == 32 ? 6 : 3)
#endif
// P buffers in shared memory: the softmax of tile G writes P into buffer
// G % kPBufs once the P V of tile G - kPBufs has read it.
#ifndef DDT_VERIFY_P_BUFS
#define DDT_VERIFY_P_BUFS (DDT_VERIFY_TILE_KEYS == 128 ? 2 : 1)
#endif
constexpr int kKStages = DDT_VERIFY_K_STAGES;      // each of the two K rings (even / odd tiles)
constexpr int kVStages = DDT_VERIFY_V_STAGES;      // V ring (feeds O += P V)
// V stage: kVKeys cache rows x 128 latent columns (this CTA's half of one N = 256
// accumulator), committed as one unit after its kVKeys / 16 MMAs.
constexpr int kVKeys = DDT_VERIFY_V_KEYS;
static_assert(kVKeys == 32 || kVKeys == 64, "V stages of 32 or 64 keys");
constexpr int kVStageBytes = kVKeys * 256;
constexpr int kQChunks = 9;                        // 8 latent chunks + 1 rope chunk
constexpr int kQBytes = kQChunks * kStageBytes;    // 64 rows x 576 bf16
constexpr int kKStagesPerTile = (kQChunks + kKStageChunks - 1) / kKStageChunks;
constexpr int kPBufBytes = kTK * 128;              // 64 rows x kTK keys bf16
constexpr int kPBufs = DDT_VERIFY_P_BUFS;
static_assert(kPBufs >= 1 && kPBufs <= 3, "one to three P buffers");
// The epilogue stages half of a CTA's bf16 output (64 rows x 256 columns) in the P
// buffers and stores it with TMA.
static_assert(kPBufs * kPBufBytes >= 64 * 256 * 2, "P buffers hold half an output tile");
constexpr int kVBlocks = kTK / kVKeys;             // V blocks per tile
constexpr int kOffQ = 0;
constexpr int kOffKRing = kOffQ + kQBytes;           // two rings of kKStages
constexpr int kOffVRing = kOffKRing + kQKIss * kKStages * kKStageBytes;
constexpr int kOffP = kOffVRing + kVStages * kVStageBytes;
constexpr int kOffRedMax = kOffP + kPBufs * kPBufBytes;  // float[2][128]
constexpr int kOffRedL = kOffRedMax + 2 * 128 * 4;     // float[128]
constexpr int kMaxSortedB = 512;  // requests ordered by length (larger B: natural order)
constexpr int kOffLen = kOffRedL + 128 * 4;            // int32[kMaxSortedB]
constexpr int kOffOrder = kOffLen + kMaxSortedB * 4;   // int32[kMaxSortedB]
constexpr int kOffBar = kOffOrder + kMaxSortedB * 4;
// barriers: two K rings' full/empty (ring g at offset g * kKStages), V ring
// full/empty, q_full, s_full[2], p_full[2], o_done, and one "all issued MMAs
// done" barrier per issuing thread (two S issuers, one O issuer).
constexpr int kBarKFull = 0;
constexpr int kBarKEmpty = kBarKFull + kQKIss * kKStages;
constexpr int kBarVFull = kBarKEmpty + kQKIss * kKStages;
constexpr int kBarVEmpty = kBarVFull + kVStages;
constexpr int kBarQ = kBarVEmpty + kVStages;
constexpr int kBarS = kBarQ + 1;           // four S buffers: S ready
constexpr int kBarSFree = kBarS + 4;       // four S buffers: read by both CTAs' softmax
constexpr int kBarP = kBarSFree + 4;      // kPBufs: P of tile G written (G % kPBufs)
constexpr int kBarO = kBarP + kPBufs;      // four: P V of tile G done (G % 4)
constexpr int kBarQKDone = kBarO + 4;      // one per S issuer
constexpr int kBarPVDone = kBarQKDone + kQKIss;
constexpr int kBarQFree = kBarPVDone + 1;  // every S issuer is done with this item's Q
constexpr int kBarOFree = kBarQFree + 1;   // both CTAs' epilogues have read O
constexpr int kNumBars = kBarOFree + 1;
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kOffAbort = kOffTmemPtr + 4;
constexpr int kSmemUsed = kOffAbort + 4;
constexpr int kSmemBytes = kSmemUsed + 1024;  // slack for 1024-byte alignment
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr int kTmemCols = 512;
constexpr int kSCols = kTK / 2;          // TMEM columns of one S buffer
constexpr int kNumS = 256 / kSCols;      // S buffers in columns [0, 256): 4 or 2
constexpr int kLogNumS = kNumS == 4 ? 2 : 1;
constexpr int kSChunks = kKH / 64;       // 64-key chunks of S per softmax thread
constexpr int kTmemS = 0;
constexpr int kTmemO = 256;  // O halves at columns 256 and 384
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kTK, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);
constexpr float kRescaleLog2 = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
}  // namespace va

struct VerifyParams {
  const int32_t* prefix_lens;
  const uint64_t* mask;
  void* out;
  float* lse;
  float* part_o;    // [num_splits][B*Q*64][512], used when num_splits > 1
  float* part_lse;  // [num_splits][B*Q*64]
  int32_t* status;
  int B, Q, capacity, num_splits, n_pairs, out_f32;
  float scale_log2;  // softmax_scale * log2(e)
  // Key range of a launch: 0 = the whole cache (prefix and tree block); 1 = the
  // prefix rows [0, P) only; 2 = the tree block [P, P+Q) only (one tile).
  int kv_mode;
  int write_partials;  // write normalised partials + lse (split-KV or a pass of a split)
  int split_base;      // partial index of this launch's split 0
};

// KV tile range [t0, t1) of split `split` for a cache of T rows.
__host__ __device__ inline void split_range(int T, int num_splits, int split, int& t0, int& t1) {
  const int n_tiles = (T + kVerifyTileKeys - 1) / kVerifyTileKeys;
  const int per = (n_tiles + num_splits - 1) / num_splits;
  t0 = split * per;
  t1 = t0 + per < n_tiles ? t0 + per : n_tiles;
}

// One work item: a pair of tree nodes of one request over one KV split.
struct WorkItem {
  int b, pair, split, P, T, end, t0, ntile, last_tile;  // end: last row + 1 of this pass
  bool bad_prefix, valid;
};

// Work index w -> item.  With `order` (requests sorted by decreasing cache
// length) the w-th item belongs to request order[w / per_req].
__device__ __forceinline__ WorkItem decode_item(const VerifyParams& p, int w, const int* order) {
  WorkItem it;
  const int per_req = p.n_pairs * p.num_splits;
  const int slot = w / per_req;
  it.b = order ? order[slot] : slot;
  const int rem = w - slot * per_req;
  it.pair = rem / p.num_splits;
  it.split = rem - it.pair * p.num_splits;
  it.P = p.prefix_lens[it.b];
  // Requests whose tree block would not fit the cache are rejected as a whole.
  it.bad_prefix = (it.P < 0) || (static_cast<int64_t>(it.P) + p.Q > p.capacity);
  it.T = it.P + p.Q;
  it.end = p.kv_mode == 1 ? it.P : it.T;
  int t0 = 0, t1 = 0;
  if (!it.bad_prefix) {
    if (p.kv_mode == 2) {
      t0 = (it.T + va::kTK - 1) / va::kTK - 1;  // the one tile ending at T holds the tree block
      t1 = t0 + 1;
    } else {
      split_range(it.end, p.num_splits, it.split, t0, t1);
    }
  }
  it.t0 = t0;
  it.ntile = t1 - t0;  // 0 for an empty split (the merge skips it)
  it.last_tile = (it.end + va::kTK - 1) / va::kTK - 1;
  it.valid = !it.bad_prefix && it.ntile > 0;
  return it;
}

// First cache row of KV tile t.  A request's last tile is shifted to end at the
// pass's last row (T, or P for a prefix pass), so no load ever reaches the rows
// past it (padding that may hold anything); its overlap with the previous tile
// is masked, and rows below 0 (fewer than kTK rows) read as zeros.
__device__ __forceinline__ int tile_start(const WorkItem& it, int t) {
  return t == it.last_tile ? it.end - va::kTK : va::kTK * t;
}

// The k-th work index of a cluster: rounds of n_clusters indices, alternating
// direction ("snake"), so that with items sorted by decreasing cost each pair
// gets a balanced mix (a static longest-first schedule).  -1 past the end.
__device__ __forceinline__ int work_index(int k, int cluster, int n_clusters, int n_items) {
  const int64_t w = static_cast<int64_t>(k) * n_clusters +
                    ((k & 1) ? (n_clusters - 1 - cluster) : cluster);
  return w < n_items ? static_cast<int>(w) : -1;
}

// Persistent kernel: each CTA pair (cluster of 2) loops over the work indices
// work_index(0, ...), work_index(1, ...), ...  Barriers, rings and tensor memory
// live across items; per-tile barrier phases follow a tile counter G that
// counts the tiles of all items a CTA has processed.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(va::kThreads, 1)
    verify_attn_kernel(const __grid_constant__ CUtensorMap tm_qlat,
                       const __grid_constant__ CUtensorMap tm_qrope,
                       const __grid_constant__ CUtensorMap tm_ckv_k,
                       const __grid_constant__ CUtensorMap tm_ckv_v,
                       const __grid_constant__ CUtensorMap tm_krope,
                       const __grid_constant__ CUtensorMap tm_out,
                       const __grid_constant__ CUtensorMap tm_f32, const VerifyParams p) {
  using namespace va;
  const uint32_t rank = cluster_ctarank();
  const int cluster = static_cast<int>(blockIdx.x >> 1);
  const int n_clusters = static_cast<int>(gridDim.x >> 1);
  const int n_items = p.B * p.n_pairs * p.num_splits;
  const int n_rounds = (n_items + n_clusters - 1) / n_clusters;
  const int Q = p.Q;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  const uint32_t sQ = base_addr + kOffQ;
  const uint32_t sKRing = base_addr + kOffKRing;
  const uint32_t sVRing = base_addr + kOffVRing;
  const uint32_t sP = base_addr + kOffP;
  float* red_max = reinterpret_cast<float*>(base + kOffRedMax);
  float* red_l = reinterpret_cast<float*>(base + kOffRedL);
  const uint32_t bars = base_addr + kOffBar;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_ptr_smem = reinterpret_cast<uint32_t*>(base + kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    // Stage and Q barriers: one arrival (the even CTA's producer, expecting the
    // bytes of both CTAs); the odd CTA's loads only add completed bytes.
    for (int s = 0; s < kQKIss * kKStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);  // the issuing thread's commit
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kNumS; ++s) {
      mbar_init(bar(kBarS + s), 1);
      mbar_init(bar(kBarSFree + s), 2);  // one arrival per CTA of the pair
    }
    for (int s = 0; s < kPBufs; ++s) mbar_init(bar(kBarP + s), 2);  // one arrival per CTA
    for (int s = 0; s < 4; ++s) mbar_init(bar(kBarO + s), 1);
    for (int g = 0; g < kQKIss; ++g) mbar_init(bar(kBarQKDone + g), 1);
    mbar_init(bar(kBarPVDone), 1);
    mbar_init(bar(kBarQFree), kQKIss);  // a commit of each S issuer
    mbar_init(bar(kBarOFree), 2);  // one arrival per CTA of the pair
    *abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == kWarpTmem) {
    tmem_alloc<2>(smem_u32(tmem_ptr_smem), kTmemCols);
    tmem_relinquish<2>();
  }
  // Requests ranked by decreasing cache length (ties by index), computed
  // redundantly by every CTA from prefix_lens: one warp per request counts, over
  // its lanes, the requests that come before it.  Invalid prefixes rank as empty.
  int* len_smem = reinterpret_cast<int*>(base + kOffLen);
  int* order_smem = reinterpret_cast<int*>(base + kOffOrder);
  const bool sorted = p.B <= kMaxSortedB;
  if (sorted) {
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
      const int P = p.prefix_lens[b];
      len_smem[b] = (P < 0 || static_cast<int64_t>(P) + Q > p.capacity) ? 0 : P + Q;
    }
    __syncthreads();
    for (int bi = warp; bi < p.B; bi += kThreads / 32) {
      const int li = len_smem[bi];
      int before = 0;
      for (int bj = lane; bj < p.B; bj += 32) {
        const int lj = len_smem[bj];
        before += (lj > li) || (lj == li && bj < bi);
      }
      before = __reduce_add_sync(0xffffffffu, before);
      if (lane == 0) order_smem[before] = bi;
    }
  }
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_ptr_smem;
  const int* order = sorted ? order_smem : nullptr;

  // Ring helper: a stage index and phase bit advancing over `n` stages.
  struct Ring {
    int stage = 0;
    uint32_t phase = 0;
    __device__ void advance(int n) {
      if (++stage == n) {
        stage = 0;
        phase ^= 1u;
      }
    }
  };
  const bool leader = rank == 0;

  // K producer g and S issuer g share ring g.
  const int qk_g = warp == kWarpKProd0 || warp == kWarpSIss0   ? 0
                   : warp == kWarpKProd1 || warp == kWarpSIss1 ? 1
                                                               : -1;
  const bool k_producer = warp == kWarpKProd0 || warp == kWarpKProd1;
  const bool s_issuer = warp == kWarpSIss0 || warp == kWarpSIss1;
  if (k_producer) {
    // ---------------------------------------------- TMA: Q and the K rings
    // Lane 0 issues; producer g loads the K stages of tiles G with G % kQKIss == g
    // (by the tile counter G), and producer 0 also loads Q.  Only the even CTA arrives on the
    // stage barriers (with the byte count of both CTAs); both CTAs' loads
    // complete bytes on them.
    if (lane == 0) {
      const int g = qk_g;
      const int key_half = static_cast<int>(rank) * kKH;
      const int full0 = kBarKFull + g * kKStages, empty0 = kBarKEmpty + g * kKStages;
      const uint32_t ring = sKRing + g * kKStages * kKStageBytes;
      const uint32_t qbar = map_to_rank(bar(kBarQ), 0);
      Ring r;
      int iter = 0;
      int64_t G = 0;
      for (int k = 0; k < n_rounds; ++k) {
        const int item = work_index(k, cluster, n_clusters, n_items);
        if (item < 0) continue;
        const WorkItem it = decode_item(p, item, order);
        if (!it.valid) continue;
        const int node = 2 * it.pair + static_cast<int>(rank);
        if (g == 0) {
          // Q of the previous item stays in use until both S issuers are done.
          if (iter > 0) mbar_wait(bar(kBarQFree), static_cast<uint32_t>((iter - 1) & 1), abort_flag);
          if (leader) mbar_arrive_expect_tx_local(bar(kBarQ), 2 * kQBytes);
          for (int c = 0; c < 8; ++c)
            tma_load_3d_pair(sQ + c * kStageBytes, &tm_qlat, qbar, 64 * c, node * 64, it.b);
          tma_load_3d_pair(sQ + 8 * kStageBytes, &tm_qrope, qbar, 0, node * 64, it.b);
        }
        for (int jj = 0; jj < it.ntile; ++jj, ++G) {
          if (static_cast<int>(G % kQKIss) != g) continue;
          const int key0 = tile_start(it, it.t0 + jj) + key_half;
          for (int sc = 0; sc < kKStagesPerTile; ++sc) {
            const int c0 = sc * kKStageChunks;
            const int nch = kQChunks - c0 < kKStageChunks ? kQChunks - c0 : kKStageChunks;
            mbar_wait(bar(empty0 + r.stage), r.phase ^ 1u, abort_flag);
            if (leader) mbar_arrive_expect_tx_local(bar(full0 + r.stage), 2 * nch * kKChunkBytes);
            const uint32_t fb = map_to_rank(bar(full0 + r.stage), 0);
            for (int u = 0; u < nch; ++u) {
              const int c = c0 + u;
              const uint32_t dst = ring + r.stage * kKStageBytes + u * kKChunkBytes;
              if (c < 8) tma_load_3d_pair(dst, &tm_ckv_k, fb, 64 * c, key0, it.b);
              else tma_load_3d_pair(dst, &tm_krope, fb, 0, key0, it.b);
            }
            r.advance(kKStages);
          }
        }
        ++iter;
      }
    }
    __syncwarp();
  } else if (warp == kWarpVProd) {
    // ------------------------------------------------------------ TMA: V ring
    if (lane == 0) {
      Ring r;
      for (int k = 0; k < n_rounds; ++k) {
        const int item = work_index(k, cluster, n_clusters, n_items);
        if (item < 0) continue;
        const WorkItem it = decode_item(p, item, order);
        if (!it.valid) continue;
        for (int jj = 0; jj < it.ntile; ++jj) {
          for (int kb = 0; kb < kVBlocks; ++kb) {
            const int key0 = tile_start(it, it.t0 + jj) + kVKeys * kb;
            for (int nh = 0; nh < 2; ++nh) {
              mbar_wait(bar(kBarVEmpty + r.stage), r.phase ^ 1u, abort_flag);
              if (leader) mbar_arrive_expect_tx_local(bar(kBarVFull + r.stage), 2 * kVStageBytes);
              const uint32_t fb = map_to_rank(bar(kBarVFull + r.stage), 0);
              const int x0 = 256 * nh + 128 * static_cast<int>(rank);
              const uint32_t dst = sVRing + r.stage * kVStageBytes;
              tma_load_3d_pair(dst, &tm_ckv_v, fb, x0, key0, it.b);
              tma_load_3d_pair(dst + kVStageBytes / 2, &tm_ckv_v, fb, x0 + 64, key0, it.b);
              r.advance(kVStages);
            }
          }
        }
      }
    }
    __syncwarp();
  } else if (s_issuer) {
    // -------------------------------------------------------- MMA: S = Q K^T
    // Issuer g takes tiles G with G % kQKIss == g; tile G goes to S buffer
    // G % kNumS.
    if (leader && lane == 0) {
      const int g = qk_g;
      const int full0 = kBarKFull + g * kKStages, empty0 = kBarKEmpty + g * kKStages;
      const uint32_t ring = sKRing + g * kKStages * kKStageBytes;
      Ring r;
      int iter = 0;
      int64_t G = 0;
      for (int k = 0; k < n_rounds; ++k) {
        const int item = work_index(k, cluster, n_clusters, n_items);
        if (item < 0) continue;
        const WorkItem it = decode_item(p, item, order);
        if (!it.valid) continue;
        mbar_wait(bar(kBarQ), static_cast<uint32_t>(iter & 1), abort_flag);
        for (int jj = 0; jj < it.ntile; ++jj, ++G) {
          if (static_cast<int>(G % kQKIss) != g) continue;
          const int sbuf = static_cast<int>(G & (kNumS - 1));
          if (G >= kNumS) {
            // S buffer sbuf is free once both CTAs' softmax has read tile G-4.
            mbar_wait(bar(kBarSFree + sbuf), static_cast<uint32_t>(((G >> kLogNumS) - 1) & 1),
                      abort_flag);
            tc_fence_after_sync();
          }
          const uint32_t d = tmem + kTmemS + static_cast<uint32_t>(kSCols * sbuf);
          for (int sc = 0; sc < kKStagesPerTile; ++sc) {
            const int c0 = sc * kKStageChunks;
            const int nch = kQChunks - c0 < kKStageChunks ? kQChunks - c0 : kKStageChunks;
            mbar_wait(bar(full0 + r.stage), r.phase, abort_flag);
            for (int u = 0; u < nch; ++u) {
              const int c = c0 + u;
              const uint32_t a0 = sQ + c * kStageBytes;
              const uint32_t b0 = ring + r.stage * kKStageBytes + u * kKChunkBytes;
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss<2>(d, smem_desc_sw128(a0 + 32 * ks, 16, 1024),
                               smem_desc_sw128(b0 + 32 * ks, 16, 1024), kIdescQK, (c | ks) != 0);
            }
            mma_commit<2>(bar(empty0 + r.stage), 0x3);
            r.advance(kKStages);
          }
          mma_commit<2>(bar(kBarS + sbuf), 0x3);
        }
        mma_commit<2>(bar(kBarQFree), 0x3);  // this issuer no longer reads this item's Q
        ++iter;
      }
      mma_commit<2>(bar(kBarQKDone + g), 0x1);
      mbar_wait(bar(kBarQKDone + g), 0, abort_flag);
    }
    __syncwarp();
  } else if (warp == kWarpPVIss) {
    // ------------------------------------------------------- MMA: O += P V
    if (leader && lane == 0) {
      Ring r;
      int iter = 0;
      int64_t G = 0;
      for (int k = 0; k < n_rounds; ++k) {
        const int item = work_index(k, cluster, n_clusters, n_items);
        if (item < 0) continue;
        const WorkItem it = decode_item(p, item, order);
        if (!it.valid) continue;
        if (iter > 0) {
          // The first P V of an item overwrites O: both CTAs' epilogues must
          // have read the previous item's O.
          mbar_wait(bar(kBarOFree), static_cast<uint32_t>((iter - 1) & 1), abort_flag);
          tc_fence_after_sync();
        }
        for (int jj = 0; jj < it.ntile; ++jj, ++G) {
          const int pb = static_cast<int>(G % kPBufs);
          mbar_wait(bar(kBarP + pb), static_cast<uint32_t>((G / kPBufs) & 1), abort_flag);
          tc_fence_after_sync();
          for (int kb = 0; kb < kVBlocks; ++kb) {
            for (int nh = 0; nh < 2; ++nh) {
              mbar_wait(bar(kBarVFull + r.stage), r.phase, abort_flag);
              const uint32_t d = tmem + kTmemO + 128u * static_cast<uint32_t>(nh);
              // P keys [kVKeys kb, + kVKeys): 64-key chunk, then 2 bytes per key in its row
              const int pk0 = kVKeys * kb;
              const uint32_t a0 = sP + pb * kPBufBytes + (pk0 >> 6) * kStageBytes + (pk0 & 63) * 2;
              const uint32_t b0 = sVRing + r.stage * kVStageBytes;
#pragma unroll
              for (int ks = 0; ks < kVKeys / 16; ++ks)
                mma_bf16_ss<2>(d, smem_desc_sw128(a0 + 32 * ks, 16, 1024),
                               smem_desc_sw128(b0 + 2048 * ks, kVStageBytes / 2, 1024), kIdescPV,
                               !(jj == 0 && kb == 0 && ks == 0));
              mma_commit<2>(bar(kBarVEmpty + r.stage), 0x3);
              r.advance(kVStages);
            }
          }
          mma_commit<2>(bar(kBarO + static_cast<int>(G & 3)), 0x3);
        }
        ++iter;
      }
      mma_commit<2>(bar(kBarPVDone), 0x1);
      mbar_wait(bar(kBarPVDone), 0, abort_flag);
    }
    __syncwarp();
  } else if (warp < 4) {
    // -------------------------------------------------------- softmax warps
    const int t = threadIdx.x;         // TMEM lane
    const int m = t & 63;              // row within this CTA (head)
    const int hf = t >> 6;             // which half of the 128-key tile / O columns
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const int W = (Q + 63) >> 6;
    const uint32_t p_full_leader0 = map_to_rank(bar(kBarP), 0);
    const uint32_t s_free_leader0 = map_to_rank(bar(kBarSFree), 0);
    const uint32_t o_free_leader = map_to_rank(bar(kBarOFree), 0);
    // P V completions are confirmed strictly in tile order (o_next = the next
    // tile to confirm) on four barriers taken by tile % 4.  The softmax waits at
    // most for tile G - kPBufs while P V can have finished at most tile G - 1,
    // so a wait never sees a barrier more than one phase ahead of it.
    int64_t o_next = 0;
    auto wait_o_through = [&](int64_t last) {
      bool waited = false;
      while (o_next <= last) {
        mbar_wait(bar(kBarO + static_cast<int>(o_next & 3)), static_cast<uint32_t>((o_next >> 2) & 1),
                  abort_flag);
        ++o_next;
        waited = true;
      }
      if (waited) tc_fence_after_sync();
    };
    int64_t G = 0;
    for (int k = 0; k < n_rounds; ++k) {
      const int item = work_index(k, cluster, n_clusters, n_items);
      if (item < 0) continue;
      const WorkItem it = decode_item(p, item, order);
      if (rank == 0 && t == 0 && it.pair == 0 && it.split == 0 && p.status)
        p.status[it.b] = it.bad_prefix ? DDT_REQ_BAD_PREFIX : DDT_REQ_OK;
      if (!it.valid) continue;
      const int b = it.b, P = it.P, T = it.T, t0 = it.t0, ntile = it.ntile, split = it.split;
      const int node = 2 * it.pair + static_cast<int>(rank);
      const bool node_valid = node < Q;
      uint64_t mw0 = 0, mw1 = 0;
      if (node_valid) {
        const uint64_t* mrow = p.mask + (static_cast<int64_t>(b) * Q + node) * W;
        mw0 = mrow[0];
        if (W > 1) mw1 = mrow[1];
      }
      float m_ref = -INFINITY;
      float l_sum = 0.f;
      float m_use = 0.f;
      for (int jj = 0; jj < ntile; ++jj, ++G) {
        const int tile = t0 + jj;
        const int sb = static_cast<int>(G & 1);              // max-exchange slot
        const int pbuf = static_cast<int>(G % kPBufs);       // P buffer
        const int sbuf = static_cast<int>(G & (kNumS - 1));  // S buffer
        mbar_wait(bar(kBarS + sbuf), static_cast<uint32_t>((G >> kLogNumS) & 1), abort_flag);
        tc_fence_after_sync();
        // This thread's keys of the tile: [kbase, kbase + kKH), in chunks of 64.
        const int kbase = tile_start(it, tile) + hf * kKH;
        // Keys below lo belong to the previous tile (a tree-block pass has none).
        // Prefix rows are visible to every node, except in a tree-block pass,
        // whose one tile may also reach prefix rows and rows below 0.
        const bool tree_pass = p.kv_mode == 2;
        const int lo = tree_pass ? INT_MIN : tile * kTK;
        // Masked raw scores of 64-key chunk sc (q . k; the scale, which the host
        // checks is positive, is applied in the exponent's FMA and to the maximum).
        auto load_chunk = [&](int sc, float (&x)[64]) {
          uint32_t r0[32], r1[32];
          const uint32_t col = tmem + lane_addr + kTmemS + static_cast<uint32_t>(kSCols * sbuf + 64 * sc);
          tmem_ld32(col, r0);
          tmem_ld32(col + 32u, r1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = __uint_as_float(r0[c]);
            x[32 + c] = __uint_as_float(r1[c]);
          }
          const int key0 = kbase + 64 * sc;
          if (tree_pass || key0 + 64 > P || key0 < lo) {  // tree block, or the shifted last tile
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int key = key0 + c;
              bool vis = !tree_pass && key < P;
              if (!vis && key >= P && key < T) {
                const int a = key - P;
                const uint64_t w = a < 64 ? mw0 : mw1;
                vis = (w >> (a & 63)) & 1ull;
              }
              if (key < lo) vis = false;
              if (!vis) x[c] = -INFINITY;
            }
          }
        };
        float x[64];
        load_chunk(0, x);
        float mx = x[0];
#pragma unroll
        for (int c = 1; c < 64; ++c) mx = fmaxf(mx, x[c]);
        // Wider tiles: the other chunks' maxima now; their scores are reloaded below.
#pragma unroll 1
        for (int sc = 1; sc < kSChunks; ++sc) {
          load_chunk(sc, x);
#pragma unroll
          for (int c = 0; c < 64; ++c) mx = fmaxf(mx, x[c]);
        }
        if (kSChunks == 1) tc_fence_before_sync();
        red_max[sb * 128 + t] = mx;
        named_barrier_sync(1, kSoftmaxThreads);
        // Every thread of this CTA has read S: release the buffer.
        if (kSChunks == 1 && t == 0) mbar_arrive_cluster(s_free_leader0 + 8u * sbuf);
        // log2 units from here: a positive scale commutes with the maximum
        mx = fmaxf(mx, red_max[sb * 128 + (t ^ 64)]) * p.scale_log2;
        float factor = 1.f;
        bool rescale = false;
        if (m_ref == -INFINITY) {
          m_ref = mx;  // nothing accumulated yet: adopt the first finite maximum
        } else if (mx > m_ref + kRescaleLog2) {
          factor = fast_exp2(m_ref - mx);
          m_ref = mx;
          l_sum *= factor;
          rescale = true;
        }
        m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
#pragma unroll 1
        for (int sc = 0; sc < kSChunks; ++sc) {
          if (sc > 0 || kSChunks > 1) load_chunk(sc, x);
          // The row sum takes the bf16-rounded weights, the values the P V product
          // multiplies, so the normalised weights sum to one exactly.
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float e0 = fast_exp2(fmaf(x[2 * c], p.scale_log2, -m_use));
            const float e1 = fast_exp2(fmaf(x[2 * c + 1], p.scale_log2, -m_use));
            pk[c] = pack_bf16x2(e0, e1);
            l_sum += __uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xffff0000u);
          }
          // The P buffer of this tile was last read by the P V of tile G - kPBufs.
          if (sc == 0) wait_o_through(G - kPBufs);
          // P tile: K-major, 128-byte swizzle, 64-key chunks of 8 KB; this thread's
          // chunk sc holds keys [hf kKH + 64 sc, + 64) of the tile.
          uint8_t* prow = base + kOffP + pbuf * kPBufBytes +
                          (hf * kSChunks + sc) * kStageBytes + m * 128;
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16) {
            uint4 v = make_uint4(pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
            *reinterpret_cast<uint4*>(prow + ((c16 ^ (m & 7)) << 4)) = v;
          }
        }
        if (kSChunks > 1) tc_fence_before_sync();
        if (jj > 0) {
          if (__any_sync(0xffffffffu, rescale)) {
            // O may be rescaled only once the P V of the previous tile is done
            // (the next one waits for this tile's P).
            wait_o_through(G - 1);
#pragma unroll 1
            for (int q = 0; q < 8; ++q) {
              uint32_t o[32];
              const uint32_t addr = tmem + lane_addr + kTmemO + 32u * q;
              tmem_ld32(addr, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
              tmem_st32(addr, o);
            }
            tmem_wait_st();
          }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        named_barrier_sync(2, kSoftmaxThreads);
        if (t == 0) {
          if (kSChunks > 1) mbar_arrive_cluster(s_free_leader0 + 8u * sbuf);  // S read twice
          mbar_arrive_cluster(p_full_leader0 + 8u * pbuf);
        }
      }
      // ----------------------------------------------------------- epilogue
      wait_o_through(G - 1);
      red_l[t] = l_sum;
      named_barrier_sync(1, kSoftmaxThreads);
      const float l_row = l_sum + red_l[t ^ 64];
      const bool empty_row = !(l_row > 0.f);
      const float inv = empty_row ? 0.f : 1.f / l_row;
      const float lse_nat = empty_row ? -INFINITY : (m_use + __log2f(l_row)) * kLn2;
      // bf16 output goes out through shared memory and TMA stores, so the
      // tensor-memory reads (and the next item's first P V) need not wait for
      // the global writes; fp32 outputs and split partials use plain stores.
      const bool tma_out = node_valid && !p.write_partials && !p.out_f32;
      if (tma_out) {
        const int row0 = (b * Q + node) * 64;
        uint8_t* stage = base + kOffP;
        const uint32_t stage_addr = base_addr + kOffP;
#pragma unroll 1
        for (int nh = 0; nh < 2; ++nh) {
#pragma unroll 1
          for (int q = 0; q < 4; ++q) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_addr + kTmemO + 128u * nh + 32u * q, o);
            tmem_wait_ld();
            // columns 256 nh + 128 hf + 32 q ..: 64-column chunk 2 hf + q / 2 of this
            // half, 16-byte units 4 (q & 1) .. + 3, 128-byte swizzle by row
            uint8_t* rowp = stage + (2 * hf + (q >> 1)) * kStageBytes + m * 128;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 val = make_uint4(
                  pack_bf16x2(__uint_as_float(o[8 * v]) * inv, __uint_as_float(o[8 * v + 1]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv));
              *reinterpret_cast<uint4*>(rowp + (((4 * (q & 1) + v) ^ (m & 7)) << 4)) = val;
            }
          }
          if (nh == 1) tc_fence_before_sync();  // every read of O is done
          fence_proxy_async_smem();
          named_barrier_sync(2, kSoftmaxThreads);
          // O has been read: the next item's first P V may overwrite it.
          if (nh == 1 && t == 0) mbar_arrive_cluster(o_free_leader);
          if (t == 0) {
            for (int c = 0; c < 4; ++c)
              tma_store_3d(&tm_out, stage_addr + c * kStageBytes, 256 * nh + 64 * c, row0, 0);
            bulk_commit_group();
            bulk_wait_group_read0();  // the staging buffer may be written again
          }
          named_barrier_sync(2, kSoftmaxThreads);
        }
        if (hf == 0 && p.lse) p.lse[static_cast<int64_t>(row0) + m] = lse_nat;
      } else if (node_valid) {
        // fp32 output, or a split's normalised partial: also staged in shared
        // memory and written with TMA tile stores (32 columns x 64 rows of fp32
        // per box, 128-byte swizzle), in four rounds of 64 rows x 128 columns.
        // Round r takes, from each thread's half row, the 64 columns
        // 256 (r / 2) + 128 hf + 64 (r % 2) + [0, 64).
        const int64_t rows_total = static_cast<int64_t>(p.B) * Q * 64;
        const int64_t row0 = (static_cast<int64_t>(b) * Q + node) * 64;
        const int grow0 = static_cast<int>(
            p.write_partials ? (split + p.split_base) * rows_total + row0 : row0);
        uint8_t* stage = base + kOffP;
        const uint32_t stage_addr = base_addr + kOffP;
#pragma unroll 1
        for (int r = 0; r < 4; ++r) {
          const int nh = r >> 1;
#pragma unroll 1
          for (int qq = 0; qq < 2; ++qq) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_addr + kTmemO + 128u * nh + 32u * (2 * (r & 1) + qq), o);
            tmem_wait_ld();
            // box 2 hf + qq, row m: 8 units of 16 bytes, 128-byte swizzle by row
            uint8_t* rowp = stage + (2 * hf + qq) * kStageBytes + m * 128;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 val = make_float4(__uint_as_float(o[4 * v]) * inv,
                                             __uint_as_float(o[4 * v + 1]) * inv,
                                             __uint_as_float(o[4 * v + 2]) * inv,
                                             __uint_as_float(o[4 * v + 3]) * inv);
              *reinterpret_cast<float4*>(rowp + ((v ^ (m & 7)) << 4)) = val;
            }
          }
          if (r == 3) tc_fence_before_sync();  // every read of O is done
          fence_proxy_async_smem();
          named_barrier_sync(2, kSoftmaxThreads);
          // O has been read: the next item's first P V may overwrite it.
          if (r == 3 && t == 0) mbar_arrive_cluster(o_free_leader);
          if (t == 0) {
            for (int k = 0; k < 4; ++k)
              tma_store_3d(&tm_f32, stage_addr + k * kStageBytes,
                           256 * nh + 128 * (k >> 1) + 64 * (r & 1) + 32 * (k & 1), grow0, 0);
            bulk_commit_group();
            bulk_wait_group_read0();  // the staging buffer may be written again
          }
          named_barrier_sync(2, kSoftmaxThreads);
        }
        if (hf == 0) {
          if (p.write_partials)
            p.part_lse[static_cast<int64_t>(split + p.split_base) * rows_total + row0 + m] = lse_nat;
          else if (p.lse) p.lse[row0 + m] = lse_nat;
        }
      } else {
        // A node past q_len (odd q_len): nothing to write; release O.
        tc_fence_before_sync();
        named_barrier_sync(2, kSoftmaxThreads);
        if (t == 0) mbar_arrive_cluster(o_free_leader);
      }
    }
    if (t == 0) bulk_wait_group0();  // this CTA's output stores have completed
  }
  // (an idle warp of the 11-warp map goes straight to the final barrier)

  // All MMAs of the pair are complete here (the softmax warps waited for the
  // last O commit, the issuer for its final commit); release tensor memory.
  __syncwarp();
  tc_fence_before_sync();
  cluster_sync();
  if (warp == kWarpTmem) {
    tc_fence_after_sync();
    tmem_dealloc<2>(tmem, kTmemCols);
  }
}

// Combine split partials: lse = log sum_s exp(lse_s), out = sum_s exp(lse_s - lse) out_s.
__global__ void __launch_bounds__(256) verify_merge_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse,
                                                           const int32_t* __restrict__ prefix_lens,
                                                           void* __restrict__ out, int out_f32,
                                                           float* __restrict__ lse, int B, int Q,
                                                           int capacity, int num_splits,
                                                           int tail) {
  const int64_t rows_total = static_cast<int64_t>(B) * Q * 64;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows_total) return;
  const int b = static_cast<int>(row / (static_cast<int64_t>(Q) * 64));
  const int P = prefix_lens[b];
  if (P < 0 || static_cast<int64_t>(P) + Q > capacity) return;
  // Partials present: the non-empty splits of the cache (whole, or with `tail`
  // the prefix rows [0, P) in num_splits - 1 splits), then the tree block's.
  const int T = tail ? P : P + Q;
  const int n_cache = tail ? num_splits - 1 : num_splits;
  auto present = [&](int s) {
    if (s >= n_cache) return true;  // the tree-block partial
    int t0, t1;
    split_range(T, n_cache, s, t0, t1);
    return t0 < t1;
  };
  // The splits' lse values lane-parallel (split s on lane s % 32), their maximum
  // and weights by warp shuffles; then the partial rows four splits at a time,
  // every load of a group issued before its accumulation.  Absent splits (never
  // written) and empty ones (lse = -inf) get weight 0 and are not read.
  float lmax = -INFINITY;
  for (int s = lane; s < num_splits; s += 32)
    if (present(s)) lmax = fmaxf(lmax, part_lse[s * rows_total + row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, off));
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
  float wsum = 0.f;
  for (int s0 = 0; s0 < num_splits; s0 += 32) {
    const int s = s0 + lane;
    float wl = 0.f;
    if (s < num_splits && present(s)) {
      const float ls = part_lse[s * rows_total + row];
      wl = (ls == -INFINITY) ? 0.f : fast_exp2((ls - lmax) * va::kLog2e);
    }
    float wsum_c = wl;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wsum_c += __shfl_xor_sync(0xffffffffu, wsum_c, off);
    wsum += wsum_c;
    const int n = num_splits - s0 < 32 ? num_splits - s0 : 32;
    for (int u0 = 0; u0 < n; u0 += 4) {
      float w[4];
      float4 v[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float wu = __shfl_sync(0xffffffffu, wl, (u0 + u) & 31);
        w[u] = u0 + u < n ? wu : 0.f;
        const float4* src = reinterpret_cast<const float4*>(
            part_o + (static_cast<int64_t>(s0 + u0 + u) * rows_total + row) * 512);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          v[u][k] = w[u] != 0.f ? src[lane + 32 * k] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc[4 * k] += w[u] * v[u][k].x;
          acc[4 * k + 1] += w[u] * v[u][k].y;
          acc[4 * k + 2] += w[u] * v[u][k].z;
          acc[4 * k + 3] += w[u] * v[u][k].w;
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  if (out_f32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + row * 512);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      dst[lane + 32 * k] = make_float4(acc[4 * k] * inv, acc[4 * k + 1] * inv, acc[4 * k + 2] * inv,
                                       acc[4 * k + 3] * inv);
  } else {
    uint2* dst = reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + row * 512);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      dst[lane + 32 * k] = make_uint2(pack_bf16x2(acc[4 * k] * inv, acc[4 * k + 1] * inv),
                                      pack_bf16x2(acc[4 * k + 2] * inv, acc[4 * k + 3] * inv));
  }
  if (lse && lane == 0) lse[row] = (wsum > 0.f) ? lmax + __logf(wsum) : -INFINITY;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D bf16 map: dims {d0 (contiguous), d1, d2}, byte strides of d1 and d2, box
// {64, box1, 1}, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box1,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, uint32_t box0 = 64) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  return fn(m, dtype, 3, const_cast<void*>(base), dims, strides, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {

// One launch of the verify kernel over key range `kv_mode` (see VerifyParams).
ddt_status launch_pass(const ddt_attn_args& a, int kv_mode, int num_splits, int write_partials,
                       int split_base, float* part_o, float* part_lse, cudaStream_t stream) {
  using namespace va;
  CUtensorMap m_qlat, m_qrope, m_ckv_k, m_ckv_v, m_krope, m_out, m_f32;
  const uint64_t rows_q = static_cast<uint64_t>(a.q_len) * 64;
  const uint64_t B = static_cast<uint64_t>(a.B);
  const uint64_t cap = static_cast<uint64_t>(a.capacity);
  bool ok = make_map(&m_qlat, a.q_lat, 512, rows_q, B, 512 * 2, rows_q * 512 * 2, 64) &&
            make_map(&m_qrope, a.q_rope, 64, rows_q, B, 64 * 2, rows_q * 64 * 2, 64) &&
            make_map(&m_ckv_k, a.c_kv, 512, cap, B, a.ckv_row_stride * 2, a.ckv_batch_stride * 2, kKH) &&
            make_map(&m_ckv_v, a.c_kv, 512, cap, B, a.ckv_row_stride * 2, a.ckv_batch_stride * 2, kVKeys) &&
            make_map(&m_krope, a.k_rope, 64, cap, B, a.kr_row_stride * 2, a.kr_batch_stride * 2, kKH);
  // bf16 output rows [B * q_len * 64, 512], stored in 64 x 64 boxes by the epilogue
  const uint64_t out_rows = static_cast<uint64_t>(a.B) * a.q_len * 64;
  if (!write_partials && a.out_dtype == DDT_BF16)
    ok = ok && make_map(&m_out, a.out, 512, out_rows, 1, 512 * 2, out_rows * 512 * 2, 64);
  else
    m_out = m_qlat;  // not read
  // fp32 rows [.., 512] stored in 32 x 64 boxes: the output, or every partial of
  // the workspace up to this pass's last split.
  const uint64_t rows_total = static_cast<uint64_t>(a.B) * a.q_len * 64;
  if (write_partials) {
    const uint64_t prow = static_cast<uint64_t>(split_base + num_splits) * rows_total;
    ok = ok && make_map(&m_f32, part_o, 512, prow, 1, 512 * 4, prow * 512 * 4, 64,
                        CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 32);
  } else if (a.out_dtype == DDT_F32) {
    ok = ok && make_map(&m_f32, a.out, 512, rows_total, 1, 512 * 4, rows_total * 512 * 4, 64,
                        CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 32);
  } else {
    m_f32 = m_qlat;  // not read
  }
  if (!ok) return DDT_ERR_INVALID_ARG;
  if (ensure_smem_limit(reinterpret_cast<const void*>(verify_attn_kernel), kSmemBytes, 1) !=
      cudaSuccess)
    return DDT_ERR_CUDA;
  VerifyParams p;
  p.prefix_lens = a.prefix_lens;
  p.mask = a.mask;
  p.out = a.out;
  p.lse = a.lse;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.status = a.status;
  p.B = a.B;
  p.Q = a.q_len;
  p.capacity = a.capacity;
  p.num_splits = num_splits;
  p.n_pairs = (a.q_len + 1) / 2;
  p.out_f32 = a.out_dtype == DDT_F32;
  p.scale_log2 = a.softmax_scale * kLog2e;
  p.kv_mode = kv_mode;
  p.write_partials = write_partials;
  p.split_base = split_base;
  // Persistent grid: at most one CTA pair per two SMs; pairs loop over items.
  const int64_t items = static_cast<int64_t>(a.B) * p.n_pairs * num_splits;
  if (items > 0x3fffffffll) return DDT_ERR_UNSUPPORTED;
  const int64_t slots = device_sm_count() / 2 > 0 ? device_sm_count() / 2 : 1;
  const int64_t grid = 2 * (items < slots ? items : slots);
  verify_attn_kernel<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, stream>>>(
      m_qlat, m_qrope, m_ckv_k, m_ckv_v, m_krope, m_out, m_f32, p);
  return cudaGetLastError() == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

ddt_status launch_merge(const ddt_attn_args& a, int num_partials, int tail, const float* part_o,
                        const float* part_lse, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.q_len * 64;
  verify_merge_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      part_o, part_lse, a.prefix_lens, a.out, a.out_dtype == DDT_F32, a.lse, a.B, a.q_len,
      a.capacity, num_partials, tail);
  return cudaGetLastError() == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace

ddt_status launch_verify_attn(const ddt_attn_args& a, int num_splits, float* part_o,
                              float* part_lse, cudaStream_t stream) {
  const ddt_status st =
      launch_pass(a, 0, num_splits, num_splits > 1, 0, part_o, part_lse, stream);
  if (st != DDT_OK || num_splits <= 1) return st;
  return launch_merge(a, num_splits, 0, part_o, part_lse, stream);
}

ddt_status launch_verify_attn_split_tail(const ddt_attn_args& a, int prefix_splits,
                                         float* part_o, float* part_lse, cudaStream_t stream) {
  ddt_status st = launch_pass(a, 1, prefix_splits, 1, 0, part_o, part_lse, stream);
  if (st != DDT_OK) return st;
  st = launch_pass(a, 2, 1, 1, prefix_splits, part_o, part_lse, stream);
  if (st != DDT_OK) return st;
  return launch_merge(a, prefix_splits + 1, 1, part_o, part_lse, stream);
}

}  // namespace ddt

namespace ddt {
// Self-test of the bounded wait: one thread waits, with a short limit, for the
// first phase of a barrier that nothing arrives at.  The wait must give up,
// record the fault bit and return; *gave_up is set to 1 when it did.
__global__ void wait_selftest_kernel(uint64_t timeout_ns, int* gave_up) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar_storage), 1);
    abort_flag = 0;
    fence_mbar_init_cluster();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool completed = mbar_wait(smem_u32(&bar_storage), 0u, &abort_flag, timeout_ns);
    if (gave_up) *gave_up = completed ? 0 : 1;
  }
}
}  // namespace ddt

extern "C" ddt_status ddt_selftest_bounded_wait(uint32_t timeout_us, int32_t* gave_up,
                                                ddt_stream_t stream) {
  if (timeout_us == 0 || timeout_us > 1000000u) return DDT_ERR_INVALID_ARG;
  ddt::wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000ull, gave_up);
  return cudaGetLastError() == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

// Diagnostic read of the library's device fault word (synchronises the device).
extern "C" ddt_status ddt_fault_flags(uint32_t* flags, int32_t reset) {
  if (!flags) return DDT_ERR_INVALID_ARG;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, ddt::ddt_fault_word, sizeof v) != cudaSuccess) return DDT_ERR_CUDA;
  *flags = v;
  if (reset) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(ddt::ddt_fault_word, &zero, sizeof zero) != cudaSuccess)
      return DDT_ERR_CUDA;
  }
  return DDT_OK;
}
