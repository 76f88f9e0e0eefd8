// MXFP4 x MXFP4 -> fp32 GEMM on the block-scaled tensor cores of sm_100a,
// consuming the quantizer's outputs directly.
//
// Source: "Oscillation-Reduced MXFP4 Training for Vision Transformers",
// abstract and rebuttal Question 2 (the forward and backward GEMMs run on
// MXFP4 operands quantized along their reduction axis; the MX format is
// supported by the Blackwell architecture).
//
//   C[m][n] = sum_k A[m][k] * B[n][k]
//
// A and B are K-major MXFP4 operands: codes [rows][K/2] with one E8M0 scale
// per 32 elements along K, the scales in the blocked order written by
// mxfp4_scales_to_blocked. A ROWS quantization of X is such an operand; so
// is a COLS quantization (the operand X^T, K along the rows of X).
//
// Design (one CTA per 128x128 tile of C, 128 threads):
//   - the K loop stages 256 K-elements (128 bytes per row) of A and B with
//     asynchronous copies into the canonical K-major layout without swizzle
//     that the matrix descriptors describe: 16-byte columns ("core matrix"
//     rows) of 8 rows, the 8-row groups 128 bytes apart (stride byte
//     offset), the 16-byte K columns 2048 bytes apart (leading byte offset);
//   - the two 512-byte blocked scale tiles of A and of B for those 256
//     elements are staged beside them and copied into tensor memory with
//     tcgen05.cp (32 lines of 16 bytes, broadcast to the four lane
//     quarters: lane 32q+i holds line i, whose bytes 4q..4q+3 are the
//     scales of row 32q+i, which is the row the lane accumulates);
//   - one thread issues four tcgen05.mma kind::mxf4 (K = 64 each, two
//     scales per row per instruction, the scale byte inside the 32-bit
//     tensor-memory cell selected by the scale-factor id) into a 128x128
//     fp32 accumulator in tensor memory, then tcgen05.commit arrives on an
//     mbarrier that every thread waits on before the stage is reused;
//   - the epilogue reads the accumulator with tcgen05.ld (warp w owns lanes
//     32w..32w+31, i.e. rows) and writes fp32 C.
// Every wait is bounded: a wait that runs out marks the tile, whose output
// is then NaN, instead of spinning forever.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "launch.cuh"
#include "mxfp4_device.cuh"
#include "tc_common.cuh"

namespace mxfp4 {

namespace {

constexpr int kGM = 128, kGN = 128;  // C tile
constexpr int kGKBytes = 128;        // K bytes of A/B per stage (256 elements)
constexpr int kGChunks = kGKBytes / 16;
constexpr int kGThreads = 128;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kAccCol = 0;    // 128 fp32 columns
constexpr uint32_t kSfaCol = 128;  // two 4-column scale tiles
constexpr uint32_t kSfbCol = 136;

struct __align__(1024) GemmSmem {
  uint8_t a[kGChunks][kGM][16];
  uint8_t b[kGChunks][kGN][16];
  uint8_t sfa[2][512];
  uint8_t sfb[2][512];
  unsigned long long mbar;
  uint32_t tmem_base;
  int failed;
};

// Instruction descriptor of kind::mxf4: E2M1 A and B (format 1), K-major
// both, N/8 at bit 17, E8M0 scales (bit 23), M/16 at bit 24; the scale
// factor ids of A (bits 29-30) and B (bits 4-5) are ORed in per MMA.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) |
                            (uint32_t(kGN >> 3) << 17) | (1u << 23) |
                            (uint32_t(kGM >> 4) << 24);

__device__ __forceinline__ void mma_mxf4(uint32_t tmem_c, uint64_t adesc,
                                         uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate, uint32_t tsfa,
                                         uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, "
      "%3, [%5], [%6], p;\n\t}\n" ::"r"(tmem_c),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa),
      "r"(tsfb));
}

__device__ __forceinline__ void copy_scales_to_tmem(uint32_t taddr,
                                                    const void* tile) {
  // 32 lines of 16 bytes, contiguous: one 8-line core matrix every 128 bytes
  const uint64_t d = smem_desc(tile, 16, 128);
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr),
               "l"(d));
}

// As copy_scales_to_tmem, with the source descriptor given.
__device__ __forceinline__ void copy_scales_desc(uint32_t taddr, uint64_t d) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d));
}

__global__ void __launch_bounds__(kGThreads)
    k_gemm_mxf4(const uint8_t* __restrict__ a, const uint8_t* __restrict__ sfa,
                const uint8_t* __restrict__ b, const uint8_t* __restrict__ sfb,
                int64_t m, int64_t n, int64_t k, float* __restrict__ c,
                int* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = int64_t(blockIdx.y) * kGM, n0 = int64_t(blockIdx.x) * kGN;
  const int64_t kbytes = k / 2;                    // bytes per operand row
  const int64_t k_tiles = (k + 127) / 128;         // blocked scale tiles along K
  const int64_t a_tile0 = (m0 / 128) * k_tiles, b_tile0 = (n0 / 128) * k_tiles;

  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    sm.failed = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&sm.tmem_base)), "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;");
  const uint32_t tmem = sm.tmem_base;

  const int64_t n_kb = (kbytes + kGKBytes - 1) / kGKBytes;
  bool ok = true;
  for (int64_t kb = 0; kb < n_kb && ok; ++kb) {
    // stage A and B: 128 rows x 8 chunks of 16 bytes each
#pragma unroll
    for (int i = 0; i < kGM * kGChunks / kGThreads; ++i) {
      const int idx = i * kGThreads + tid;
      const int row = idx / kGChunks, ch = idx % kGChunks;
      const int64_t kofs = kb * kGKBytes + 16 * ch;
      const bool va = m0 + row < m && kofs < kbytes;
      const bool vb = n0 + row < n && kofs < kbytes;
      cp_async16(&sm.a[ch][row][0], a + (va ? (m0 + row) * kbytes + kofs : 0), va);
      cp_async16(&sm.b[ch][row][0], b + (vb ? (n0 + row) * kbytes + kofs : 0), vb);
    }
    // stage the scale tiles of this K block: 2 tiles of A, 2 of B
    {
      const int which = tid >> 6, j = (tid >> 5) & 1, line = tid & 31;
      const int64_t kt = 2 * kb + j;
      const bool v = kt < k_tiles;
      const uint8_t* src = which == 0 ? sfa + (a_tile0 + kt) * 512 + 16 * line
                                      : sfb + (b_tile0 + kt) * 512 + 16 * line;
      uint8_t* dst = which == 0 ? &sm.sfa[j][16 * line] : &sm.sfb[j][16 * line];
      cp_async16(dst, v ? src : (which == 0 ? sfa : sfb), v);
    }
    cp_async_commit();
    cp_async_wait<0>();
    // make this thread's shared-memory writes visible to the tensor cores
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        copy_scales_to_tmem(tmem + kSfaCol + 4 * j, &sm.sfa[j][0]);
        copy_scales_to_tmem(tmem + kSfbCol + 4 * j, &sm.sfb[j][0]);
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t sf_id = 2u * (s & 1);
        const uint32_t idesc = kIdesc | (sf_id << 29) | (sf_id << 4);
        const uint32_t tsfa = (tmem + kSfaCol + 4 * (s >> 1)) | (sf_id << 30);
        const uint32_t tsfb = (tmem + kSfbCol + 4 * (s >> 1)) | (sf_id << 30);
        const uint64_t ad = smem_desc(&sm.a[2 * s][0][0], kGM * 16, 128);
        const uint64_t bd = smem_desc(&sm.b[2 * s][0][0], kGN * 16, 128);
        mma_mxf4(tmem + kAccCol, ad, bd, idesc, (kb > 0 || s > 0) ? 1u : 0u,
                 tsfa, tsfb);
      }
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
          ::"r"(smem_u32(&sm.mbar)));
    }
    ok = wait_parity(&sm.mbar, uint32_t(kb & 1), kAccWaitLimit);
    if (!ok) {
      atomicExch(&sm.failed, 1);
      // drain: the MMAs just issued still read shared memory and write the
      // accumulator; let them finish before anything is reused or freed
      wait_parity(&sm.mbar, uint32_t(kb & 1));
    }
    __syncthreads();
    ok = sm.failed == 0;
  }

  // epilogue: warp w reads accumulator rows 32w..32w+31
  asm volatile("tcgen05.fence::after_thread_sync;");
  const int64_t row = m0 + 32 * warp + lane;
  const bool failed = sm.failed != 0;
#pragma unroll 1
  for (int cb = 0; cb < kGN / 32; ++cb) {
    uint32_t v[32];
    const uint32_t taddr = tmem + (uint32_t(32 * warp) << 16) + kAccCol + 32 * cb;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, "
        "%7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, "
        "%21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]),
          "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]),
          "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
          "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
          "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
          "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    if (row < m) {
      float* out = c + row * n + n0 + 32 * cb;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n0 + 32 * cb + j < n)
          out[j] = failed ? __uint_as_float(kNaNf32) : __uint_as_float(v[j]);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;");
  __syncthreads();
  report_failure(status, &sm.failed);
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 ::"r"(tmem), "r"(kTmemCols));
}

// ---------------------------------------------------------------------------
// Pipelined, persistent version (K a multiple of 256): one CTA per SM loops
// over 128 x 256 tiles of C. TMA loads in the 128-byte swizzled K-major
// layout through a kPS-stage ring of full/empty mbarriers; warp roles:
//   warp 0: one thread issues the tensor-memory-access (TMA) loads of A and B
//           and the bulk copies of their scale tiles into a free stage, tile
//           after tile without pause;
//   warp 1: allocates tensor memory; one thread waits until the epilogue has
//           read the accumulator, then per stage copies the scales into
//           tensor memory and issues one M = 128, N = 256 MMA per K = 64
//           step, whose completion (tcgen05.commit) frees the stage, and
//           finally commits the tile to the epilogue;
//   warps 2-9: epilogue, two warps per lane quarter (32 accumulator rows),
//           128 columns each held in registers: the accumulator is released
//           as soon as it is read and the stores of C overlap the next
//           tile's main loop.
// ---------------------------------------------------------------------------

constexpr int kPS = 4;            // pipeline stages
// kind::mxf4 instruction descriptor for M = 128, N = 256
constexpr uint32_t kIdescN256 = (1u << 7) | (1u << 10) | (uint32_t(256 >> 3) << 17) |
                                (1u << 23) | (uint32_t(kGM >> 4) << 24);
constexpr int kPN = 256;          // C tile columns
constexpr int kPEpiWarps = 8;
constexpr int kPThreads = 32 * (2 + kPEpiWarps);
constexpr uint32_t kPTmemCols = 512;
constexpr uint32_t kPSfCol = 256;  // per stage: 8 SFA columns, then 16 SFB

// Tile order: groups of kGroupM row tiles of C, each group swept across all
// column tiles before the next (the last group may be narrower). The CTAs
// running at one time then cover about kGroupM x (CTAs / kGroupM) tiles, so
// their A and B panels stay in L2 while they stream through K.
constexpr int64_t kGroupM = 16;
__device__ __forceinline__ void tile_coords(int64_t tile, int64_t m_tiles,
                                            int64_t nt_n, int64_t& m0,
                                            int64_t& n0, int64_t rows = kGM) {
  const int64_t per_group = kGroupM * nt_n;
  const int64_t g = tile / per_group, r = tile % per_group;
  const int64_t rest = m_tiles - g * kGroupM;
  const int64_t gm = rest < kGroupM ? rest : kGroupM;
  m0 = (g * kGroupM + r % gm) * rows;
  n0 = (r / gm) * kPN;
}

struct __align__(1024) PipeSmem {
  uint8_t a[kPS][kGM][128];       // 128 rows x 128 bytes, 128B-swizzled
  uint8_t b[kPS][kPN][128];
  uint8_t epi[kPEpiWarps][32][64];   // per epilogue warp: 32 rows x 16 fp32, 64B-swizzled
  uint8_t sfa[kPS][2][512];       // 2 blocked tiles (256 K elements)
  uint8_t sfb[kPS][2][2][512];    // [128-row block][K tile]
  unsigned long long full[kPS], empty[kPS], acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int failed;
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], "
      "%2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// TMA store of a 2-D box from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y,
                                             const void* src) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(smem_u32(src))
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until every committed bulk store of this thread has finished reading
// its shared-memory source.
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}


__global__ void __launch_bounds__(kPThreads, 1)
    k_gemm_mxf4_pipe(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c, bool tma_store,
                     const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb,
                     int64_t m, int64_t n, int64_t k, float* __restrict__ c,
                     int* __restrict__ status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte swizzle wants 1024-byte aligned tiles: align the base by
  // hand (the launch requests 1 KB of slack)
  PipeSmem& sm = *reinterpret_cast<PipeSmem*>(
      smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t k_tiles = k / 128;
  const int64_t n_kb = k / 256;
  const int64_t n_row_tiles = (n + 127) / 128;
  const int64_t m_tiles = (m + kGM - 1) / kGM;
  const int64_t n_col_tiles = (n + kPN - 1) / kPN;
  const int64_t n_tiles = m_tiles * n_col_tiles;

  if (tid == 0) {
    for (int s = 0; s < kPS; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.full[s])));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.empty[s])));
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.acc_full)));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&sm.acc_empty)),
                 "r"(kPEpiWarps));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.drain)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    sm.failed = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&sm.tmem_base)), "r"(kPTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;");
  const uint32_t tmem = sm.tmem_base;

  // CTA i takes tiles i, i + grid, ... in the grouped order of tile_coords.
  // The two issuing threads keep their per-stage work small: the stage index
  // and phase advance by increments, operand addresses and descriptors are
  // computed once and offset by constants, and the MMA loop is unrolled over
  // the stages when every tile starts at stage 0 (K/256 a multiple of kPS).
  if (warp == 0) {
    if (lane == 0) {
      uint32_t s = 0, ph = 0;
      // stages with a load issued, and the phase parity of each one's last
      // load: before the CTA ends, every load must have landed
      uint32_t issued = 0, last_ph = 0;
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        int64_t m0, n0;
        tile_coords(tile, m_tiles, n_col_tiles, m0, n0);
        const int64_t rb = n0 / 128;
        const bool half1 = rb + 1 < n_row_tiles;
        const uint32_t bytes = kGM * 128 + kPN * 128 + 1024 + (half1 ? 2048 : 1024);
        // blocked scales: 512-byte tiles of 128 rows x 4 groups, K tiles first
        const uint8_t* pa = sfa + (m0 / 128) * k_tiles * 512;
        const uint8_t* pb0 = sfb + rb * k_tiles * 512;
        const uint8_t* pb1 = pb0 + k_tiles * 512;
        bool stop = false;
        for (int64_t kb = 0; kb < n_kb; ++kb) {
          if (!wait_parity_or_failed<false>(&sm.empty[s], ph ^ 1u, &sm.failed)) {
            atomicExch(&sm.failed, 1);
            stop = true;
            break;
          }
          issued |= 1u << s;
          last_ph = (last_ph & ~(1u << s)) | (ph << s);
          expect_tx(&sm.full[s], bytes);
          tma_load_2d(&sm.a[s][0][0], &tm_a, int(kb) * 128, int(m0), &sm.full[s]);
          tma_load_2d(&sm.b[s][0][0], &tm_b, int(kb) * 128, int(n0), &sm.full[s]);
          bulk_load(&sm.sfa[s][0][0], pa + kb * 1024, 1024, &sm.full[s]);
          bulk_load(&sm.sfb[s][0][0][0], pb0 + kb * 1024, 1024, &sm.full[s]);
          if (half1) bulk_load(&sm.sfb[s][1][0][0], pb1 + kb * 1024, 1024, &sm.full[s]);
          if (++s == kPS) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (stop || failed_flag(&sm.failed)) break;
      }
      // drain (immediate unless a wait ran out)
      for (uint32_t st = 0; st < kPS; ++st)
        if ((issued >> st) & 1u) wait_parity(&sm.full[st], (last_ph >> st) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // scale factors in tensor memory: row r of an operand in lane r % 32,
      // 32-bit column r / 32 (A: 4 columns per K tile; B, 256 rows: 8, its
      // two 128-row tiles side by side), one byte per 32-element group;
      // tensor-core operations of one thread run in order, so the next
      // stage's copy may reuse the columns
      const uint32_t sf = tmem + kPSfCol;
      const uint64_t a_d0 = smem_desc_sw128(&sm.a[0][0][0]);
      const uint64_t b_d0 = smem_desc_sw128(&sm.b[0][0][0]);
      const uint64_t sfa_d0 = smem_desc(&sm.sfa[0][0][0], 16, 128);
      const uint64_t sfb_d0 = smem_desc(&sm.sfb[0][0][0][0], 16, 128);
      // descriptor start-address steps (16-byte units): one stage of A, of
      // B, of A's and of B's scales, one 512-byte scale tile; the K = 64
      // step inside a 128-byte swizzle row is 32 bytes
      constexpr uint32_t kAStep = (kGM * 128) >> 4, kBStep = (kPN * 128) >> 4;
      constexpr uint32_t kSfaStep = 1024 >> 4, kSfbStep = 2048 >> 4, kSfTile = 512 >> 4;
      auto issue_stage = [&](uint32_t st, bool first) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          copy_scales_desc(sf + 4 * j, sfa_d0 + (st * kSfaStep + j * kSfTile));
          copy_scales_desc(sf + 8 + 8 * j, sfb_d0 + (st * kSfbStep + j * kSfTile));
          copy_scales_desc(sf + 8 + 8 * j + 4, sfb_d0 + (st * kSfbStep + (2 + j) * kSfTile));
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint32_t sf_id = 2u * (t & 1);
          const uint32_t idesc = kIdescN256 | (sf_id << 29) | (sf_id << 4);
          const uint32_t tsfa = (sf + 4 * (t >> 1)) | (sf_id << 30);
          const uint32_t tsfb = (sf + 8 + 8 * (t >> 1)) | (sf_id << 30);
          mma_mxf4(tmem, a_d0 + (st * kAStep + 2 * t), b_d0 + (st * kBStep + 2 * t), idesc,
                   (first && t == 0) ? 0u : 1u, tsfa, tsfb);
        }
        commit_to(&sm.empty[st]);
      };
      uint32_t s = 0, ph = 0;
      int64_t ti = 0;
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++ti) {
        // the epilogue has read the previous tile's accumulator
        if (!wait_parity_or_failed<false>(&sm.acc_empty, uint32_t(ti & 1) ^ 1u, &sm.failed) ||
            failed_flag(&sm.failed)) {
          atomicExch(&sm.failed, 1);
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;");
        bool ok = true;
        if (n_kb % kPS == 0) {
          for (int64_t kb4 = 0; kb4 < n_kb && ok; kb4 += kPS) {
#pragma unroll
            for (int st = 0; st < kPS; ++st) {
              if (!wait_parity_or_failed<false>(&sm.full[st], ph, &sm.failed)) {
                ok = false;
                break;
              }
              asm volatile("tcgen05.fence::after_thread_sync;");
              issue_stage(uint32_t(st), kb4 == 0 && st == 0);
            }
            ph ^= 1u;
          }
        } else {
          for (int64_t kb = 0; kb < n_kb; ++kb) {
            if (!wait_parity_or_failed<false>(&sm.full[s], ph, &sm.failed)) {
              ok = false;
              break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;");
            issue_stage(s, kb == 0);
            if (++s == kPS) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) atomicExch(&sm.failed, 1);
        commit_to(&sm.acc_full);
        if (!ok) break;
      }
      // drain: every MMA and scale copy issued has completed before the
      // stages or the tensor memory can go away
      commit_to(&sm.drain);
      if (!wait_parity(&sm.drain, 0)) atomicExch(&sm.failed, 1);
    }
    __syncwarp();
  } else {
    // epilogue: 8 warps, two per lane quarter, each taking 128 of the 256
    // columns into registers; the accumulator is released as soon as they
    // are read, and the stores overlap the next tile's main loop
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    int64_t ti = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++ti) {
      int64_t m0, n0;
      tile_coords(tile, m_tiles, n_col_tiles, m0, n0);
      // after a failure the warp skips the tensor memory and the barriers
      // and writes NaN over the rest of its tiles
      const bool ok = __all_sync(0xFFFFFFFFu, !failed_flag(&sm.failed) &&
                                                  wait_parity(&sm.acc_full, uint32_t(ti & 1),
                                                              kAccWaitLimit));
      if (!ok) atomicExch(&sm.failed, 1);
      uint32_t v[128];
      if (ok) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        const uint32_t tbase = tmem + (uint32_t(32 * q) << 16) + 128u * uint32_t(half);
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t* d = v + 32 * cb;
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, "
              "%7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, "
              "%21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
              : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]),
                "=r"(d[5]), "=r"(d[6]), "=r"(d[7]), "=r"(d[8]), "=r"(d[9]),
                "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]),
                "=r"(d[15]), "=r"(d[16]), "=r"(d[17]), "=r"(d[18]), "=r"(d[19]),
                "=r"(d[20]), "=r"(d[21]), "=r"(d[22]), "=r"(d[23]), "=r"(d[24]),
                "=r"(d[25]), "=r"(d[26]), "=r"(d[27]), "=r"(d[28]), "=r"(d[29]),
                "=r"(d[30]), "=r"(d[31])
              : "r"(tbase + 32u * uint32_t(cb)));
        }
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;");
        __syncwarp();
        if (lane == 0)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&sm.acc_empty))
                       : "memory");
      }
      if (!ok || failed_flag(&sm.failed)) {
#pragma unroll
        for (int j = 0; j < 128; ++j) v[j] = kNaNf32;
      }
      const int64_t row = m0 + 32 * q + lane;
      const int64_t col0 = n0 + 128 * half;
      if (tma_store) {
        // 8 boxes of 32 rows x 16 fp32 through this warp's 2 KB staging
        // tile: lane r writes row r, 16-byte chunk j at chunk position
        // j ^ ((r / 2) % 4) (the 64-byte swizzle the tensor map undoes;
        // conflict-free), then lane 0 stores the box; the tile is rewritten
        // once the store has read it
        uint8_t* tile = &sm.epi[warp - 2][0][0];
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {
          if (lane == 0) bulk_wait_read();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(tile + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(v[16 * cb + 4 * j], v[16 * cb + 4 * j + 1],
                           v[16 * cb + 4 * j + 2], v[16 * cb + 4 * j + 3]);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0 && col0 + 16 * cb < n && m0 + 32 * q < m)
            tma_store_2d(&tm_c, int(col0 + 16 * cb), int(m0 + 32 * q), tile);
        }
      } else if (row < m && col0 < n) {
        float* out = c + row * n + col0;
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (col0 + j < n) out[j] = __uint_as_float(v[j]);
      }
    }
  }
  if (warp >= 2 && lane == 0) bulk_wait_all();  // C stores complete
  asm volatile("tcgen05.fence::before_thread_sync;");
  __syncthreads();
  report_failure(status, &sm.failed);
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 ::"r"(tmem), "r"(kPTmemCols));
}


// ---------------------------------------------------------------------------
// Thread-block clusters (the fused GEMM's shared quantization)
// ---------------------------------------------------------------------------

// This CTA's rank in its cluster, the cluster's index and the number of
// clusters of a one-dimensional grid.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// The address in the cluster's shared window of the byte at shared address
// a of the CTA of rank `rank`.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t a, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(rank));
  return d;
}
// Every thread of every CTA of the cluster (release, then acquire).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// wait_parity_or_failed for a barrier that other CTAs of the cluster also
// complete (acquire at cluster scope).
__device__ __forceinline__ bool wait_cluster_or_failed(unsigned long long* bar,
                                                       uint32_t parity, const int* failed) {
  const uint32_t a = smem_u32(bar);
  for (long long i = 0; i < kWaitLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if ((i & 63) == 63 && failed_flag(failed)) return false;
  }
  return false;
}
// The code words v (4, 8 or 16 bytes) to p, in one store.
__device__ __forceinline__ void put_words(uint8_t* p, const uint32_t (&v)[1]) {
  *reinterpret_cast<uint32_t*>(p) = v[0];
}
__device__ __forceinline__ void put_words(uint8_t* p, const uint32_t (&v)[2]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(v[0], v[1]);
}
__device__ __forceinline__ void put_words(uint8_t* p, const uint32_t (&v)[4]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(v[0], v[1], v[2], v[3]);
}
// A plain store to another CTA's shared memory (a from cluster_addr).
__device__ __forceinline__ void st_cluster(uint32_t a, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
// Asynchronous stores into the shared memory of another CTA of the cluster
// (a and the mbarrier bar both from cluster_addr, bar in the same CTA as
// a): the bytes count towards bar's transaction count when they land, and
// nothing waits for them here.
__device__ __forceinline__ void st_async(uint32_t a, uint32_t v, uint32_t bar) {
  asm volatile("st.async.weak.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
               ::"r"(a), "r"(v), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async(uint32_t a, const uint32_t (&v)[1], uint32_t bar) {
  st_async(a, v[0], bar);
}
__device__ __forceinline__ void st_async(uint32_t a, const uint32_t (&v)[2], uint32_t bar) {
  asm volatile(
      "st.async.weak.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];"
      ::"r"(a), "r"(v[0]), "r"(v[1]), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void st_async(uint32_t a, const uint32_t (&v)[4], uint32_t bar) {
  asm volatile(
      "st.async.weak.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, "
      "%4}, [%5];" ::"r"(a),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(bar)
      : "memory");
}
// commit_to on the mbarrier at the same offset in every CTA of cta_mask.
__device__ __forceinline__ void commit_to_cluster(unsigned long long* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask));
}

// ---------------------------------------------------------------------------
// Forward GEMM with the activation quantized in the load stage:
//   C = Q_D(X) B^T,  X bf16 [M][K] in 1x32 groups along K, nearest-even
// (source: "Oscillation-Reduced MXFP4 Training for Vision Transformers",
// rebuttal Question 2: the forward GEMM on Q_D(X) and Q_D(W)). B is a
// K-major MXFP4 operand as above (the pre-quantized weight). Same tiles
// (128 x 256), tile order and MMA issue as k_gemm_mxf4_pipe; A never exists
// in global memory unless asked for:
//   warp 0:   one thread issues the TMA loads of bf16 X in slots of
//             128-byte-swizzled boxes of 64 columns into a kQX-deep ring;
//   warp 2:   one thread loads B's codes and scales into the operand stage
//             (its own thread, so that X keeps streaming while B waits for
//             a free stage);
//   warp 1:   tensor memory; one thread waits for both halves of a stage
//             (B landed, A quantized) and issues the MMAs as above;
//   warps 3-18 (workers): during a tile's main loop the threads quantize
//             the row groups of every X slot (one or a part of a group
//             each) with the rows quantizer's arithmetic (bf16 absmax, OCP
//             scale byte, the product with 2^-e formed as one exact
//             mixed-precision multiply of the bf16 input, nearest-even
//             E2M1: bit-identical codes), write the code bytes into the
//             operand stage at their place in the 128-byte-swizzled K-major
//             layout of the MMA and the scale byte into the blocked tile
//             that tcgen05.cp copies to tensor memory, then release the X
//             slot; once the first stage of the next tile is quantized (the
//             MMAs of the previous one have drained meanwhile) the workers
//             read the previous tile's accumulator (warp w: lane quarter
//             w % 4, 64 columns) and store it. The CTAs of the first column
//             tile can also write the codes and scales to global memory in
//             the ROWS layout of mxfp4_quantize.
// RT is the number of X rows a tile covers: 128, or 64 when 128-row tiles
// would leave SMs idle; then the MMA still spans 128 rows, of which the
// last 64 are left over in shared memory and never stored.
//
// Clusters (CS = 2 or 4 CTAs): every column tile needs the whole quantized
// A of its rows, so without sharing X is re-read and re-quantized once per
// column tile. The CS CTAs of a cluster take the same rows and CS adjacent
// column tiles; each loads and quantizes RT / CS of the rows of every
// K = 256 stage and sends the codes and scale words to the operand stage of
// every CTA of the cluster with asynchronous distributed-shared-memory
// stores, whose bytes complete that CTA's stage barrier (armed by its MMA
// thread with the stage's byte count): no fence or arrival on the workers'
// path. A stage is written once every CTA's MMAs have finished reading it:
// each MMA thread's commit arrives on that barrier in every CTA of the
// cluster. Work per CTA and X traffic drop by CS.
// ---------------------------------------------------------------------------

constexpr int kQWorkers = 16;
constexpr int kQFirstWorker = 3;   // warps 0-2: X loads, MMA, B loads
constexpr int kQThreads = 32 * (kQFirstWorker + kQWorkers);

// How a K = 256 stage (8 groups of 32 per row) is shared out for tiles of
// RT rows in clusters of CS CTAs: each CTA quantizes kRows = RT / CS of the
// rows; an X slot holds kSlotG of the 8 groups of those rows (kRows x 64
// kSlotG bytes, boxes of 64 columns), so a stage takes kSlots slots; kTpg
// adjacent worker threads share one group, each with kChunks of its four
// 16-byte chunks (8 elements each). Without a cluster the 512 workers take
// one group each (the slot holds 4 groups of 128 rows, or all 8 of 64);
// in a cluster a slot holds the whole stage of a CTA's rows.
template <int RT, int CS>
struct QaSplit {
  static constexpr int kRows = RT / CS;
  static constexpr int kSlotG = CS > 1 ? 8 : (512 / RT < 8 ? 512 / RT : 8);
  static constexpr int kSlots = 8 / kSlotG;
  static constexpr int kTpg = 32 * kQWorkers / (kRows * kSlotG);
  static constexpr int kChunks = 4 / kTpg;
  static_assert(kRows % 16 == 0 && kSlotG % 2 == 0 && kTpg >= 1 && kTpg <= 4 &&
                    kRows * kSlotG * kTpg == 32 * kQWorkers,
                "work split");
};

// Shared memory of k_gemm_qa<RT, CS> (byte offsets from a 1024-aligned
// base): the X ring (kQX slots), the A ring (kQA stages of RT rows x 128
// code bytes), the B ring (kQB stages of 256 rows x 128 bytes), the blocked
// scale tiles of A and B per stage, the mbarriers. With RT = 64 the MMA
// still reads 128 rows of A: a stage's last 64 rows are the next 8 KB of
// shared memory (the next A stage, or the first B stage), whose products
// land in accumulator rows that are never stored; the 8 KB saved per stage
// buy a deeper B ring.
template <int RT, int CS>
struct QaLayout {
  static constexpr uint32_t kXSlot = QaSplit<RT, CS>::kRows * QaSplit<RT, CS>::kSlotG * 64;
  static constexpr uint32_t kAStage = RT * 128;
  // ring depths: without a cluster 96 KB of X slots, two A stages and two B
  // stages (three with 64-row tiles); in a cluster the X slots shrink with
  // the CTA's share of the rows and the space goes to deeper A and B rings,
  // which hide the longer trip of a stage through the cluster
  static constexpr int kQX = CS > 1 ? (49152 / kXSlot > 2 ? 49152 / kXSlot : 2) : 98304 / kXSlot;
  static constexpr int kQB = CS > 1 ? (RT == 64 ? 4 : 3) : (RT == 64 ? 3 : 2);
  static constexpr uint32_t kFixed = kQX * kXSlot + kQB * (kPN * 128 + 2048) + 2048;
  static constexpr int kQA =
      CS > 1 ? (kFixed + 4 * (kAStage + 1024) <= 226 * 1024 ? 4 : 3) : 2;
  static constexpr uint32_t kBStage = kPN * 128;
  static constexpr uint32_t kX = 0;
  static constexpr uint32_t kA = kX + kQX * kXSlot;
  static constexpr uint32_t kB = kA + kQA * kAStage;
  static constexpr uint32_t kSfa = kB + kQB * kBStage;
  static constexpr uint32_t kSfb = kSfa + kQA * 1024;
  static constexpr uint32_t kBar = kSfb + kQB * 2048;
  // barriers: full_b, empty_b [kQB]; full_a, empty_a [kQA]; x_full, x_empty
  // [kQX]; acc_full, acc_empty, drain; then tmem_base and the failure flag
  static constexpr uint32_t kFullB = kBar, kEmptyB = kFullB + 8 * kQB;
  static constexpr uint32_t kFullA = kEmptyB + 8 * kQB, kEmptyA = kFullA + 8 * kQA;
  static constexpr uint32_t kXFull = kEmptyA + 8 * kQA, kXEmpty = kXFull + 8 * kQX;
  static constexpr uint32_t kAccFull = kXEmpty + 8 * kQX, kAccEmpty = kAccFull + 8;
  static constexpr uint32_t kDrain = kAccEmpty + 8, kTmemBase = kDrain + 8;
  static constexpr uint32_t kFailed = kTmemBase + 4;
  static constexpr uint32_t kBytes = kFailed + 4;
  static_assert(kXSlot % 1024 == 0 && kA % 1024 == 0 && kB % 1024 == 0 &&
                    kAStage % 1024 == 0,
                "swizzle atoms");
  static_assert(kA + (kQA - 1) * kAStage + kGM * 128 <= kSfa, "A padding rows in bounds");
};

// The part `part` (of TPG) of one 32-element group of X: its 4 / TPG
// 16-byte chunks of bf16 (chunk 4 part / TPG + j in w[j]), quantized as the
// rows quantizer does: code words out[j] (element i of the chunk in nibble
// i) and the group's scale byte sb; the TPG threads of a group are adjacent
// lanes and combine their maxima with shuffles. Nearest rounding: the
// scaled values v = x 2^-e come from one mixed-precision product of the
// bf16 input with 2^-e (a normal bf16 power of two for every byte the OCP
// rule gives), rounded once, the fp32 product the rows quantizer forms
// after widening. Stochastic rounding (SR): bf16x8_sr_word, the rows
// quantizer's pair form, with the group's counter base kh (its first pair
// index, keyed) and the chunk's index in the group.
template <bool SR, int TPG>
__device__ __forceinline__ void qa_quantize_part(const uint4 (&w)[4 / TPG], int part,
                                                 uint32_t kh, uint32_t& sb,
                                                 uint32_t (&out)[4 / TPG]) {
  constexpr int NC = 4 / TPG;
  uint32_t mx[2 * NC];
#pragma unroll
  for (int j = 0; j < NC; ++j) {
    mx[2 * j] = bf16x2_absmax_nan(w[j].x, w[j].y);
    mx[2 * j + 1] = bf16x2_absmax_nan(w[j].z, w[j].w);
  }
#pragma unroll
  for (int h = NC; h >= 1; h /= 2)
#pragma unroll
    for (int i = 0; i < h; ++i) mx[i] = bf16x2_absmax_nan(mx[i], mx[i + h]);
#pragma unroll
  for (int o = 1; o < TPG; o *= 2)
    mx[0] = bf16x2_absmax_nan(mx[0], __shfl_xor_sync(0xFFFFFFFFu, mx[0], o));
  const uint32_t mm = mx[0] & 0x7FFF7FFFu;
  sb = scale_byte(max(mm << 16, mm & 0xFFFF0000u));
  const unsigned short s16 = bf16_inv_scale(sb);
  if (SR) {
    const uint32_t sat2 = bf16x2_six_scale(sb);
#pragma unroll
    for (int j = 0; j < NC; ++j)
      out[j] = bf16x8_sr_word<false>(reinterpret_cast<const uint32_t*>(&w[j]), s16, sat2, kh,
                                     uint32_t(NC * part + j));
  } else {
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const uint32_t* q = reinterpret_cast<const uint32_t*>(&w[j]);
      float v[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        v[2 * t] = bf16lo_mul(q[t], s16);
        v[2 * t + 1] = bf16hi_mul(q[t], s16);
      }
      out[j] = e2m1x8_rn(v);
    }
  }
  if (sb == 0xFFu)
#pragma unroll
    for (int j = 0; j < NC; ++j) out[j] = 0;
}

template <int RT, int CS, bool SR>
__global__ void __launch_bounds__(kQThreads, 1)
    k_gemm_qa(const __grid_constant__ CUtensorMap tm_x,
              const __grid_constant__ CUtensorMap tm_b,
              const uint8_t* __restrict__ sfb, int64_t m, int64_t n, int64_t k, RngKey key,
              float* __restrict__ c, uint8_t* __restrict__ a_codes,
              uint8_t* __restrict__ a_scales, int* __restrict__ status) {
  using L = QaLayout<RT, CS>;
  using P = QaSplit<RT, CS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* const sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  auto bar = [&](uint32_t off, int i) {
    return reinterpret_cast<unsigned long long*>(sm + off) + i;
  };
  int* const failed = reinterpret_cast<int*>(sm + L::kFailed);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this CTA's place: cluster `cid` of `ncl` works on tiles cid, cid + ncl, ..
  const uint32_t rank = CS > 1 ? cluster_rank() : 0u;
  const int64_t cid = CS > 1 ? int64_t(cluster_index()) : int64_t(blockIdx.x);
  const int64_t ncl = CS > 1 ? int64_t(cluster_count()) : int64_t(gridDim.x);
  const int64_t k_tiles = k / 128;
  const int64_t n_kb = k / 256;
  const int64_t n_row_tiles = (n + 127) / 128;
  const int64_t m_tiles = (m + RT - 1) / RT;
  const int64_t n_col_groups = ((n + kPN - 1) / kPN + CS - 1) / CS;
  const int64_t n_tiles = m_tiles * n_col_groups;
  // tile t of the cluster: X rows from m0, this CTA's C columns from n0;
  // first: the cluster's columns start at 0
  auto coords = [&](int64_t t, int64_t& m0, int64_t& n0, bool& first) {
    int64_t q0;
    tile_coords(t, m_tiles, n_col_groups, m0, q0, RT);
    first = q0 == 0;
    n0 = q0 * CS + int64_t(rank) * kPN;
  };
  // a wait ran out: stop this CTA and, through their flags, the others of
  // the cluster (which would wait for its stages)
  auto fail = [&]() {
    atomicExch(failed, 1);
    if (CS > 1)
      for (uint32_t d = 0; d < uint32_t(CS); ++d)
        if (d != rank) st_cluster(cluster_addr(smem_u32(failed), d), 1u);
  };

  if (tid == 0) {
    auto init = [&](uint32_t off, int i, uint32_t count) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar(off, i))),
                   "r"(count));
    };
    for (int i = 0; i < L::kQB; ++i) init(L::kFullB, i, 1), init(L::kEmptyB, i, 1);
    // a stage is full once every worker warp of the CTA has stored its
    // share (in a cluster also: once its MMA thread has armed it with the
    // other CTAs' bytes and those have come in), and free once every CTA's
    // MMAs have read it
    for (int i = 0; i < L::kQA; ++i)
      init(L::kFullA, i, kQWorkers + (CS > 1 ? 1 : 0)), init(L::kEmptyA, i, CS);
    for (int i = 0; i < L::kQX; ++i) init(L::kXFull, i, 1), init(L::kXEmpty, i, kQWorkers);
    init(L::kAccFull, 0, 1);
    init(L::kAccEmpty, 0, kQWorkers);
    init(L::kDrain, 0, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    *failed = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(sm + L::kTmemBase)), "r"(kPTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;");
  // every CTA's barriers are initialised before any other CTA arrives on them
  if (CS > 1) cluster_sync_all();
  const uint32_t tmem = *reinterpret_cast<const uint32_t*>(sm + L::kTmemBase);

  if (warp == 0 || warp == 2) {
    // warp 0: X into its ring; warp 2: B into its ring. Two threads, so
    // that neither ring waits on the other's consumer.
    if (lane == 0) {
      const bool loads_x = warp == 0;
      const int ring = loads_x ? L::kQX : L::kQB;
      uint32_t s = 0, ph = 0;
      // slots with a load issued, and the phase parity of each one's last
      // load: every load lands before the CTA ends
      uint32_t issued = 0, last = 0;
      bool stop = false;
      for (int64_t tile = cid; tile < n_tiles && !stop; tile += ncl) {
        int64_t m0, n0;
        bool first;
        coords(tile, m0, n0, first);
        // B's rows from n0; none when this column tile of the cluster lies
        // past n (then the stage is marked full without a load: the MMAs
        // read whatever the stage holds into accumulator columns that are
        // never stored)
        const int64_t rb = n0 / 128;
        const bool half0 = rb < n_row_tiles, half1 = rb + 1 < n_row_tiles;
        const uint32_t bbytes = L::kBStage + (half1 ? 2048 : 1024);
        for (int64_t kb = 0; kb < n_kb && !stop; ++kb) {
          for (int h = 0; h < (loads_x ? P::kSlots : 1); ++h) {
            if (!wait_parity_or_failed<false>(bar(loads_x ? L::kXEmpty : L::kEmptyB, s),
                                              ph ^ 1u, failed)) {
              stop = true;
              break;
            }
            issued |= 1u << s;
            last = (last & ~(1u << s)) | (ph << s);
            if (loads_x) {
              unsigned long long* full = bar(L::kXFull, s);
              expect_tx(full, L::kXSlot);
              // this CTA's rows (from m0 + rank kRows), the slot's kSlotG
              // groups in boxes of 64 columns
              const int64_t e0 = kb * 256 + 32 * P::kSlotG * h;
#pragma unroll
              for (int j = 0; j < P::kSlotG / 2; ++j)
                tma_load_2d(sm + L::kX + s * L::kXSlot + j * P::kRows * 128, &tm_x,
                            int((e0 + 64 * j) * 2), int(m0 + rank * P::kRows), full);
            } else {
              unsigned long long* full = bar(L::kFullB, s);
              uint8_t* sfb_s = sm + L::kSfb + s * 2048;
              if (half0) {
                expect_tx(full, bbytes);
                tma_load_2d(sm + L::kB + s * L::kBStage, &tm_b, int(kb) * 128, int(n0), full);
                bulk_load(sfb_s, sfb + (rb * k_tiles + 2 * kb) * 512, 1024, full);
                if (half1)
                  bulk_load(sfb_s + 1024, sfb + ((rb + 1) * k_tiles + 2 * kb) * 512, 1024,
                            full);
              } else {
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(full))
                             : "memory");
              }
            }
            if (++s == uint32_t(ring)) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        if (failed_flag(failed)) stop = true;
      }
      if (stop) fail();
      // drain (immediate unless a wait ran out)
      for (int st = 0; st < ring; ++st)
        if ((issued >> st) & 1u)
          wait_parity(bar(loads_x ? L::kXFull : L::kFullB, st), (last >> st) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t sf = tmem + kPSfCol;
      const uint64_t a_d0 = smem_desc_sw128(sm + L::kA);
      const uint64_t b_d0 = smem_desc_sw128(sm + L::kB);
      const uint64_t sfa_d0 = smem_desc(sm + L::kSfa, 16, 128);
      const uint64_t sfb_d0 = smem_desc(sm + L::kSfb, 16, 128);
      constexpr uint32_t kAStep = L::kAStage >> 4, kBStep = L::kBStage >> 4;
      constexpr uint32_t kSfaStep = 1024 >> 4, kSfbStep = 2048 >> 4, kSfTile = 512 >> 4;
      uint32_t sa = 0, pha = 0, sb = 0, phb = 0;
      int64_t ti = 0;
      bool ok = true;
      // in a cluster, every A stage expects from the other CTAs their rows
      // (RT / CS each) of 128 code bytes and two 4-byte scale words
      constexpr uint32_t kStageBytes = (CS - 1) * P::kRows * (128 + 8);
      if (CS > 1)
        for (int i = 0; i < L::kQA; ++i) expect_tx(bar(L::kFullA, i), kStageBytes);
      for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl, ++ti) {
        if (!wait_parity_or_failed<false>(bar(L::kAccEmpty, 0), uint32_t(ti & 1) ^ 1u,
                                          failed) ||
            failed_flag(failed)) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;");
        for (int64_t kb = 0; kb < n_kb; ++kb) {
          if (!wait_parity_or_failed<false>(bar(L::kFullB, sb), phb, failed) ||
              !(CS > 1 ? wait_cluster_or_failed(bar(L::kFullA, sa), pha, failed)
                      : wait_parity_or_failed<false>(bar(L::kFullA, sa), pha, failed))) {
            ok = false;
            break;
          }
          if (CS > 1) {
            // arm the stage's next use; the other CTAs' asynchronous stores
            // that filled this one are ordered before the tensor cores' reads
            expect_tx(bar(L::kFullA, sa), kStageBytes);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          }
          asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            copy_scales_desc(sf + 4 * j, sfa_d0 + (sa * kSfaStep + j * kSfTile));
            copy_scales_desc(sf + 8 + 8 * j, sfb_d0 + (sb * kSfbStep + j * kSfTile));
            copy_scales_desc(sf + 8 + 8 * j + 4, sfb_d0 + (sb * kSfbStep + (2 + j) * kSfTile));
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const uint32_t sf_id = 2u * (t & 1);
            const uint32_t idesc = kIdescN256 | (sf_id << 29) | (sf_id << 4);
            const uint32_t tsfa = (sf + 4 * (t >> 1)) | (sf_id << 30);
            const uint32_t tsfb = (sf + 8 + 8 * (t >> 1)) | (sf_id << 30);
            mma_mxf4(tmem, a_d0 + (sa * kAStep + 2 * t), b_d0 + (sb * kBStep + 2 * t), idesc,
                     (kb == 0 && t == 0) ? 0u : 1u, tsfa, tsfb);
          }
          // the A stage is shared: free it in every CTA of the cluster
          if (CS > 1)
            commit_to_cluster(bar(L::kEmptyA, sa), uint16_t((1u << CS) - 1u));
          else
            commit_to(bar(L::kEmptyA, sa));
          commit_to(bar(L::kEmptyB, sb));
          if (++sa == uint32_t(L::kQA)) {
            sa = 0;
            pha ^= 1u;
          }
          if (++sb == uint32_t(L::kQB)) {
            sb = 0;
            phb ^= 1u;
          }
        }
        if (!ok) fail();
        commit_to(bar(L::kAccFull, 0));
      }
      if (!ok) fail();
      // drain: every MMA and scale copy issued has completed
      commit_to(bar(L::kDrain, 0));
      if (!wait_parity(bar(L::kDrain, 0), 0)) fail();
    }
    __syncwarp();
  } else {
    // workers: thread qt works on part qt % kTpg of group g of row rl of
    // every X slot (item qt / kTpg: g kRows + rl alone, rl 8 + g in a
    // cluster, where the four groups of a scale word sit in adjacent
    // lanes); rl is row r of the tile (row rank kRows + rl in a cluster);
    // warp w stores lane quarter w % 4, columns 64 ((w - 3) / 4) of every
    // accumulator
    const int qt = tid - 32 * kQFirstWorker;
    const int part = qt % P::kTpg;
    const int item = qt / P::kTpg;
    const int rl = CS > 1 ? item / 8 : item % P::kRows;
    const int g = CS > 1 ? item % 8 : item / P::kRows;  // box g / 2, half g % 2 of it
    const int r = int(rank) * P::kRows + rl;
    const uint32_t sw = uint32_t(rl & 7);              // = r & 7
    const uint8_t* xrow = sm + L::kX + (g >> 1) * P::kRows * 128 + rl * 128;
    const int q = warp & 3;
    const int cblk = (warp - kQFirstWorker) >> 2;
    uint32_t s = 0, ph = 0, xs = 0, xph = 0;
    bool ok = true;
    int64_t pend_ti = -1, pend_m0 = 0, pend_n0 = 0;

    // the accumulator of tile ti (origin m0, n0) to C; after a failure,
    // NaN without touching tensor memory or the barriers
    auto drain_tile = [&](int64_t ti, int64_t m0, int64_t n0) {
      const bool got = __all_sync(0xFFFFFFFFu, !failed_flag(failed) &&
                                                   wait_parity(bar(L::kAccFull, 0),
                                                               uint32_t(ti & 1),
                                                               kAccWaitLimit));
      if (!got) fail();
      uint32_t v[64];
      if (got) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        const uint32_t tbase = tmem + (uint32_t(32 * q) << 16) + 64u * uint32_t(cblk);
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
          uint32_t* d = v + 32 * cb;
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, "
              "%7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, "
              "%21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
              : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]),
                "=r"(d[5]), "=r"(d[6]), "=r"(d[7]), "=r"(d[8]), "=r"(d[9]),
                "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]),
                "=r"(d[15]), "=r"(d[16]), "=r"(d[17]), "=r"(d[18]), "=r"(d[19]),
                "=r"(d[20]), "=r"(d[21]), "=r"(d[22]), "=r"(d[23]), "=r"(d[24]),
                "=r"(d[25]), "=r"(d[26]), "=r"(d[27]), "=r"(d[28]), "=r"(d[29]),
                "=r"(d[30]), "=r"(d[31])
              : "r"(tbase + 32u * uint32_t(cb)));
        }
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;");
        __syncwarp();
        if (lane == 0)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(
                           smem_u32(bar(L::kAccEmpty, 0)))
                       : "memory");
      }
      if (!got || failed_flag(failed)) {
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = kNaNf32;
      }
      const int64_t row = m0 + 32 * q + lane;
      const int64_t col0 = n0 + 64 * cblk;
      if (32 * q + lane < RT && row < m && col0 < n) {
        float* out = c + row * n + col0;
        if (col0 + 64 <= n && (n & 3) == 0) {
#pragma unroll
          for (int j = 0; j < 64; j += 4)
            *reinterpret_cast<uint4*>(out + j) = make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (col0 + j < n) out[j] = __uint_as_float(v[j]);
        }
      }
    };

    int64_t ti = 0;
    for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl, ++ti) {
      int64_t m0, n0;
      bool first;
      coords(tile, m0, n0, first);
      const int64_t row = m0 + r;
      const bool to_global = first && a_codes != nullptr && row < m;
      for (int64_t kb = 0; kb < n_kb; ++kb) {
        // the A stage is free once the MMAs of its last use completed (in
        // every CTA of the cluster)
        if (!__all_sync(0xFFFFFFFFu,
                        CS > 1 ? wait_cluster_or_failed(bar(L::kEmptyA, s), ph ^ 1u, failed)
                               : wait_parity_or_failed<false>(bar(L::kEmptyA, s), ph ^ 1u,
                                                             failed))) {
          ok = false;
          break;
        }
        uint8_t* const a_s = sm + L::kA + s * L::kAStage;
        uint8_t* const sfa_s = sm + L::kSfa + s * 1024;
        for (int h = 0; h < P::kSlots; ++h) {
          if (!__all_sync(0xFFFFFFFFu,
                          wait_parity_or_failed<false>(bar(L::kXFull, xs), xph, failed))) {
            ok = false;
            break;
          }
          const uint8_t* xr = xrow + xs * L::kXSlot;
          uint4 w[P::kChunks];
#pragma unroll
          for (int j = 0; j < P::kChunks; ++j)
            w[j] = *reinterpret_cast<const uint4*>(
                xr + (((4 * (g & 1) + P::kChunks * part + j) ^ sw) << 4));
          // the group within the stage's 8
          const int G = P::kSlotG * h + g;
          uint32_t kh = 0;
          if (SR) {  // the group's first pair index, row-major over X
            const uint64_t p0 = uint64_t(row * (k / 32) + kb * 8 + G) * 16u;
            kh = inner_key(key, uint32_t(p0 >> 32)) + uint32_t(p0);
          }
          uint32_t scb, code[P::kChunks];
          qa_quantize_part<SR, P::kTpg>(w, part, kh, scb, code);
          const uint32_t code_off = r * 128 + ((uint32_t(G) ^ sw) << 4) + 4 * P::kChunks * part;
          const uint32_t sc_off = 512 * (G >> 2) + 16 * (r & 31) + 4 * (r >> 5);
          if constexpr (CS > 1) {
            // the scale word of groups 4t .. 4t+3 (t = G / 4) of row r,
            // gathered in the lane of group 4t, part 0
            uint32_t word = scb << (8 * (G & 3));
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, P::kTpg);
            word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2 * P::kTpg);
            const bool word_lane = (G & 3) == 0 && part == 0;
            // into this CTA's operand stage, and asynchronously into every
            // other CTA's, whose stage barrier counts the bytes
            put_words(a_s + code_off, code);
            if (word_lane) *reinterpret_cast<uint32_t*>(sfa_s + sc_off) = word;
            const uint32_t fa = smem_u32(bar(L::kFullA, s));
            const uint32_t ca = smem_u32(a_s + code_off), wa = smem_u32(sfa_s + sc_off);
#pragma unroll
            for (int j = 1; j < CS; ++j) {
              const uint32_t d = (rank + uint32_t(j)) % uint32_t(CS);
              const uint32_t bd = cluster_addr(fa, d);
              st_async(cluster_addr(ca, d), code, bd);
              if (word_lane) st_async(cluster_addr(wa, d), word, bd);
            }
          } else {
            put_words(a_s + code_off, code);
            if (part == 0) sfa_s[sc_off + (G & 3)] = uint8_t(scb);
          }
          if (to_global) {
            put_words(a_codes + row * (k / 2) + kb * 128 + 16 * G + 4 * P::kChunks * part, code);
            if (part == 0) a_scales[row * (k / 32) + kb * 8 + G] = uint8_t(scb);
          }
          // release the X slot after the stores that depend on every value
          // loaded from it: a thread's arrival does not wait for its shared
          // loads to return, so releasing right after issuing them let the
          // next TMA load into the slot overwrite data still being read
          __syncwarp();
          if (lane == 0)
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(
                             smem_u32(bar(L::kXEmpty, xs)))
                         : "memory");
          if (++xs == uint32_t(L::kQX)) {
            xs = 0;
            xph ^= 1u;
          }
        }
        if (!ok) break;
        // this CTA's share of the stage was written through the generic
        // proxy; the tensor cores read it through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(
                           smem_u32(bar(L::kFullA, s)))
                       : "memory");
        if (++s == uint32_t(L::kQA)) {
          s = 0;
          ph ^= 1u;
        }
        // the previous tile's accumulator, once this tile's first stage is
        // on its way: its MMAs have drained meanwhile
        if (kb == 0 && pend_ti >= 0) {
          drain_tile(pend_ti, pend_m0, pend_n0);
          pend_ti = -1;
        }
      }
      if (!ok) break;
      pend_ti = ti, pend_m0 = m0, pend_n0 = n0;
    }
    if (!ok) fail();
    if (pend_ti >= 0) drain_tile(pend_ti, pend_m0, pend_n0);
  }
  // after a timeout, asynchronous stores of this cluster may still be on
  // their way to a CTA that stopped waiting for them: let them land before
  // any CTA of the cluster can leave (they take microseconds)
  if (CS > 1 && failed_flag(failed))
    for (int i = 0; i < 100; ++i) __nanosleep(1000);
  asm volatile("tcgen05.fence::before_thread_sync;");
  __syncthreads();
  // no CTA leaves while another of the cluster may still store into its
  // shared memory or arrive on its barriers
  if (CS > 1) cluster_sync_all();
  report_failure(status, failed);
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 ::"r"(tmem), "r"(kPTmemCols));
}

}  // namespace

namespace {

// 2-D map over K-major codes [rows][k/2]: boxes of 128 bytes x box_rows,
// 128-byte swizzle, zero fill outside the tensor.
bool encode_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t k,
                      uint32_t box_rows) {
  return encode_rows_sw128(map, codes, rows, k / 2, box_rows);
}

// 2-D map over fp32 C [m][n] for the epilogue's stores: boxes of 32 rows x
// 16 columns, 64-byte swizzle (the staging tiles' layout).
bool encode_c_map(CUtensorMap* map, float* c, int64_t m, int64_t n) {
  auto enc = tensor_map_encoder();
  if (!enc || n % 4) return false;
  const cuuint64_t dims[2] = {cuuint64_t(n), cuuint64_t(m)};
  const cuuint64_t strides[1] = {cuuint64_t(n) * 4};
  const cuuint32_t box[2] = {16, 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, c, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm_mxf4(const uint8_t* a, const uint8_t* a_scales,
                             const uint8_t* b, const uint8_t* b_scales,
                             int64_t m, int64_t n, int64_t k, float* c,
                             int* status, cudaStream_t s) {
  if (k % 256 == 0) {
    CUtensorMap ma, mb, mc;
    if (encode_codes_map(&ma, a, m, k, kGM) && encode_codes_map(&mb, b, n, k, kPN)) {
      const bool tma_store = encode_c_map(&mc, c, m, n);
      if (!tma_store) mc = ma;  // unused
      constexpr size_t smem = sizeof(PipeSmem) + 1024;
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(k_gemm_mxf4_pipe),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(smem));
      if (e != cudaSuccess) return e;
      const int64_t tiles = ((m + kGM - 1) / kGM) * ((n + kPN - 1) / kPN);
      const int grid = persistent_grid(reinterpret_cast<const void*>(k_gemm_mxf4_pipe),
                                       kPThreads, smem, tiles);
      k_gemm_mxf4_pipe<<<grid, kPThreads, smem, s>>>(ma, mb, mc, tma_store, a_scales,
                                                     b_scales, m, n, k, c, status);
      return cudaGetLastError();
    }
  }
  // Two CTAs per SM at most: each holds 256 of the SM's 512 tensor-memory
  // columns, so the shared memory request keeps a third from being resident
  // (and blocking in its allocation).
  constexpr size_t smem = 100 * 1024;
  static_assert(sizeof(GemmSmem) <= smem, "gemm smem");
  cudaError_t e = cudaFuncSetAttribute(
      reinterpret_cast<const void*>(k_gemm_mxf4),
      cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned((n + kGN - 1) / kGN), unsigned((m + kGM - 1) / kGM));
  k_gemm_mxf4<<<grid, kGThreads, smem, s>>>(a, a_scales, b, b_scales, m, n, k, c, status);
  return cudaGetLastError();
}

namespace {

template <int RT, int CS, bool SR>
cudaError_t gemm_qa_impl(const void* x, int64_t m, int64_t n, int64_t k, RngKey key,
                         const uint8_t* b, const uint8_t* b_scales, float* c, uint8_t* a_codes,
                         uint8_t* a_scales, int* status, cudaStream_t s) {
  // X as a byte array [m][2k] for the TMA: 128-byte boxes of 64 bf16
  CUtensorMap mx, mb;
  if (!encode_rows_sw128(&mx, x, m, 2 * k, QaSplit<RT, CS>::kRows) ||
      !encode_codes_map(&mb, b, n, k, kPN))
    return cudaErrorInvalidValue;
  constexpr size_t smem = QaLayout<RT, CS>::kBytes + 1024;
  static_assert(smem <= 227 * 1024, "fused GEMM shared memory");
  auto kern = k_gemm_qa<RT, CS, SR>;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(kern),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  // tiles of a cluster: RT rows x CS column tiles
  const int64_t tiles = ((m + RT - 1) / RT) * (((n + kPN - 1) / kPN + CS - 1) / CS);
  if (CS == 1) {
    const int grid = persistent_grid(reinterpret_cast<const void*>(kern), kQThreads, smem, tiles);
    kern<<<grid, kQThreads, smem, s>>>(mx, mb, b_scales, m, n, k, key, c, a_codes, a_scales,
                                       status);
    return cudaGetLastError();
  }
  // persistent clusters: as many as can be resident at once
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // the number of resident clusters, asked once per device (the query
  // costs more host time than the launch)
  static int resident[64] = {};
  int clusters = dev >= 0 && dev < 64 ? resident[dev] : 0;
  if (clusters < 1) {
    cfg.gridDim = dim3(unsigned(sms / CS * CS));
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64) resident[dev] = clusters;
  }
  cfg.gridDim = dim3(unsigned((tiles < clusters ? tiles : clusters) * CS));
  return cudaLaunchKernelEx(&cfg, kern, mx, mb, b_scales, m, n, k, key, c, a_codes, a_scales,
                            status);
}

template <int RT, bool SR>
cudaError_t gemm_qa_cluster(int cs, const void* x, int64_t m, int64_t n, int64_t k, RngKey key,
                            const uint8_t* b, const uint8_t* b_scales, float* c,
                            uint8_t* a_codes, uint8_t* a_scales, int* status, cudaStream_t s) {
  if (cs == 4)
    return gemm_qa_impl<RT, 4, SR>(x, m, n, k, key, b, b_scales, c, a_codes, a_scales, status, s);
  if (cs == 2)
    return gemm_qa_impl<RT, 2, SR>(x, m, n, k, key, b, b_scales, c, a_codes, a_scales, status, s);
  return gemm_qa_impl<RT, 1, SR>(x, m, n, k, key, b, b_scales, c, a_codes, a_scales, status, s);
}

}  // namespace

cudaError_t launch_gemm_qa(const void* x, int64_t m, int64_t n, int64_t k, bool sr,
                           uint64_t seed, const uint8_t* b, const uint8_t* b_scales, float* c,
                           uint8_t* a_codes, uint8_t* a_scales, int* status,
                           cudaStream_t s) {
  if (k % 256) return cudaErrorInvalidValue;
  const RngKey key = make_key(seed, 0);
  // clusters of up to 4 CTAs share the quantization of their rows over as
  // many column tiles; 64-row tiles where they all run at once (a 64-row
  // tile takes about 0.8 of a 128-row one, so 128-row tiles win as soon as
  // the 64-row ones would need a second wave)
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t col_tiles = (n + kPN - 1) / kPN;
  const int cs = col_tiles >= 4 ? 4 : (col_tiles >= 2 ? 2 : 1);
  const int64_t ctas64 = ((m + 63) / 64) * ((col_tiles + cs - 1) / cs) * cs;
  if (ctas64 <= sms)
    return sr ? gemm_qa_cluster<64, true>(cs, x, m, n, k, key, b, b_scales, c, a_codes,
                                          a_scales, status, s)
              : gemm_qa_cluster<64, false>(cs, x, m, n, k, key, b, b_scales, c, a_codes,
                                           a_scales, status, s);
  return sr ? gemm_qa_cluster<128, true>(cs, x, m, n, k, key, b, b_scales, c, a_codes, a_scales,
                                         status, s)
            : gemm_qa_cluster<128, false>(cs, x, m, n, k, key, b, b_scales, c, a_codes,
                                          a_scales, status, s);
}

}  // namespace mxfp4
