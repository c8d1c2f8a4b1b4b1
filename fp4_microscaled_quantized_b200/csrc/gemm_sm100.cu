// Block-scaled FP4 GEMM on the 5th-generation tensor cores (sm_100a).
//
// D[M x N] = (A . SFA) (B . SFB)^T * (tA * tB), both operands K-major ("TN"),
// FP32 accumulation in tensor memory -- the Quartet page's stage-2 kernel
// D = C + (A x SFA) . (B x SFB); NVFP4 uses kind::mxf4nvf4 with E4M3 scales per
// 16, MXFP4 kind::mxf4 with E8M0 scales per 32.  An optional epilogue applies
// the Quartet backward correction dx = 16/9 H32^-1(dx_q (.) (1 - M)) (the 16/9
// is the product of the two 4/3 tensor scales).
//
// Structure: persistent CTAs (one per SM), 128 x 256 output tiles, a 3-stage
// shared-memory ring fed by TMA (codes, 128-byte swizzle) and bulk copies
// (scale atoms, already in the tensor-core layout), warp roles:
//   warp 0  TMA producer          warp 1  MMA issuer (one thread)
//   warp 2  TMEM allocator        warps 4-7  epilogue (TMEM -> smem -> TMA store)
//   warps 8-11  scale-factor stagers: each writes its TMEM lane quadrant of the
//   scales with tcgen05.st into one of two TMEM buffers, so the MMA issue queue
//   holds only MMAs (copying scales with tcgen05.cp from the MMA thread
//   serialises them with the MMAs and halves throughput).
// Every mbarrier wait is bounded; on timeout the kernel records
// FP4_ERR_TIMEOUT, stops issuing work, frees its TMEM and returns.
#include <cuda.h>
#include <atomic>
#include <cstdlib>
#include <mutex>

#include "../../include/fp4.h"
#include "device_common.cuh"

namespace fp4 {

int* status_ptr();
int num_sms();

namespace gemm {

constexpr int BM = 128, BN = 256, BK = 256;         // BK in FP4 elements (128 bytes)
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK / 2;                 // 16 KB
constexpr int B_BYTES = BN * BK / 2;                 // 32 KB
constexpr int SFA_BYTES = 4 * 512;                   // up to 4 atoms (NVFP4)
constexpr int SFB_BYTES = 8 * 512;                   // 2 row blocks x 4 atoms
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int STG_BYTES = BM * 128;                  // epilogue staging: 128 rows x 128 bytes
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 2 * STG_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr int THREADS = 384;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns: the accumulator, then NSF scale-factor buffers (SFA 16 + SFB
// 32 columns each) so the stagers run ahead of the MMAs.
constexpr uint32_t ACC_COL = 0, SF_COL = 256, SF_BUF_COLS = 48, SFB_OFF = 16;
constexpr int NSF = 4;                               // scale-factor TMEM buffers (256 + 4 x 48 <= 512 columns)
constexpr unsigned long long WAIT_LIMIT = 4000000000ull;  // ~2 s of SM clocks

enum : int { OUT_F32 = 0, OUT_BF16 = 1 };

struct Params {
  int64_t M, N, K;
  const uint8_t* sfa;   // swizzled scale atoms of A
  const uint8_t* sfb;
  int64_t nkb;          // atoms per 128-row block (= ceil(K / g / 4))
  const float* ta;
  const float* tb;
  void* D;
  const uint8_t* mask;  // epilogue clip mask (M x N bits) or null
  int* status;
  int raster;           // CTA-pair tile order (tile_coords2)
};

// ----------------------------------------------------------- PTX helpers --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: false (and the abort flag raised) when the limit is hit.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  if (mbar_try(b, parity)) return true;
  const unsigned long long t0 = clock64();
  while (true) {
    if (mbar_try(b, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > WAIT_LIMIT) {
      *abort_flag = 1;
      flag_status(status, ST_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// TMA store of a staged tile (bulk-group completion) and its bookkeeping.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// OR of a predicate over the 128 epilogue threads (named barrier 1).
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// K-major operand tile with the 128-byte swizzle: 8-row core groups 1024 B
// apart (SBO), one swizzle atom along K (LBO unused), descriptor version 1.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFF);
  d |= uint64_t(1024 >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

template <int FMT>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t sfa, uint32_t sfb, uint32_t acc) {
  if (FMT == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
  }
}

// Instruction descriptor of the block-scaled MMA: E2M1 x E2M1, both K-major,
// N and M, scale type (0 = UE4M3, 1 = UE8M0) and the scale byte ids.
__device__ __forceinline__ uint32_t idesc(int fmt, int n, int m, uint32_t sfa_id, uint32_t sfb_id) {
  uint32_t d = 0;
  d |= (sfb_id & 3u) << 4;
  d |= 1u << 7;                    // A: E2M1
  d |= 1u << 10;                   // B: E2M1
  d |= uint32_t(n >> 3) << 17;
  d |= uint32_t(fmt == 1 ? 0 : 1) << 23;
  d |= uint32_t(m >> 4) << 24;
  d |= (sfa_id & 3u) << 29;
  return d;
}

// The MMAs of one full k-tile (NK of K = 64), unrolled: the operand
// descriptors advance by 32 bytes (2 in their 16-byte address field) per MMA,
// the scale-factor TMEM addresses by one atom (4 columns of A, 8 of B; MXFP4
// takes two MMAs per atom, bytes 0-1 then 2-3), and only the first MMA of a
// tile's first k-tile overwrites the accumulator.
template <int FMT, int NK, bool PAIR = false>
__device__ __forceinline__ void mma_ktile(uint32_t acc, uint64_t ad, uint64_t bd, uint32_t sfbase, uint32_t idesc0,
                                          bool accumulate);

// The same load without its wait (several loads, then one tcgen05.wait::ld).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Tile order: groups of 16 M-blocks sweep all N-blocks, so the CTAs resident
// at one time share A rows and B rows in L2.
__device__ __forceinline__ void tile_coords(int64_t t, int64_t nm, int64_t nn, int64_t& mb, int64_t& nb) {
  const int64_t G = 16;
  int64_t per_group = G * nn;
  int64_t g = t / per_group, r = t % per_group;
  int64_t gm = nm - g * G < G ? nm - g * G : G;
  mb = g * G + r % gm;
  nb = r / gm;
}

// ---------------------------------------------------------------- kernel --
template <int FMT, int OUT, int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
           const __grid_constant__ CUtensorMap map_d, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sSFA = sB + STAGES * B_BYTES;
  uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;
  uint8_t* sStage = sSFB + STAGES * SFB_BYTES;         // 1024-byte aligned (stage sizes are)
  uint64_t* full = reinterpret_cast<uint64_t*>(sStage + 2 * STG_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* sf_full = acc_empty + 1;
  uint64_t* sf_empty = sf_full + NSF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + NSF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nm = (p.M + BM - 1) / BM, nn = (p.N + BN - 1) / BN, ntiles = nm * nn;
  const int64_t nkt = (p.K + BK - 1) / BK;
  constexpr int G = FMT == 1 ? 16 : 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 128);
    for (int b = 0; b < NSF; ++b) { mbar_init(&sf_full[b], 128); mbar_init(&sf_empty[b], 1); }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer --
    int s = 0;
    uint32_t ph = 0;
    for (int64_t t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
      int64_t mb, nb;
      tile_coords(t, nm, nn, mb, nb);
      for (int64_t kt = 0; kt < nkt; ++kt) {
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.status)) break;
        const int kel = int(p.K - kt * BK < BK ? p.K - kt * BK : BK);
        const int n_mma = kel / 64;
        const int atoms = FMT == 1 ? n_mma : (n_mma + 1) / 2;       // per 128-row block
        const int64_t atom0 = kt * (BK / G / 4);
        const int64_t nrb = (p.N + 127) / 128;
        const int rb_b = (nb * 2 + 1 < nrb) ? 2 : 1;
        const uint32_t sf_bytes = uint32_t(atoms) * 512u * uint32_t(1 + rb_b);
        mbar_expect_tx(&full[s], uint32_t(A_BYTES + B_BYTES) + sf_bytes);
        tma_load_2d(sA + s * A_BYTES, &map_a, int(kt * (BK / 2)), int(mb * BM), &full[s]);
        tma_load_2d(sB + s * B_BYTES, &map_b, int(kt * (BK / 2)), int(nb * BN), &full[s]);
        bulk_load(sSFA + s * SFA_BYTES, p.sfa + (mb * p.nkb + atom0) * 512, atoms * 512u, &full[s]);
        for (int r = 0; r < rb_b; ++r)
          bulk_load(sSFB + s * SFB_BYTES + r * 4 * 512, p.sfb + ((nb * 2 + r) * p.nkb + atom0) * 512,
                    atoms * 512u, &full[s]);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------- MMA issue --
    // Walks this CTA's (tile, k-tile) sequence; k-tile i uses operand stage
    // i % STAGES and scale buffer i % 2.
    int s = 0, buf = 0;
    uint32_t ph = 0, acc_ph = 0;
    uint32_t sph = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok && t < ntiles && !*abort_flag; t += gridDim.x) {
      if (!mbar_wait(acc_empty, acc_ph ^ 1, abort_flag, p.status)) break;
      tc_fence_after();
      for (int64_t kt = 0; kt < nkt; ++kt) {
        if (!mbar_wait(&full[s], ph, abort_flag, p.status)) { ok = false; break; }
        if (!mbar_wait(&sf_full[buf], sph, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const int kel = int(p.K - kt * BK < BK ? p.K - kt * BK : BK);
        const int n_mma = kel / 64;
        const uint64_t ad = desc_sw128(smem_u32(sA + s * A_BYTES)), bd = desc_sw128(smem_u32(sB + s * B_BYTES));
        const uint32_t sfbase = tmem + SF_COL + SF_BUF_COLS * uint32_t(buf);
        if (n_mma == BK / 64) {
          mma_ktile<FMT, BK / 64>(tmem + ACC_COL, ad, bd, sfbase, idesc(FMT, BN, BM, 0, 0), kt > 0);
        } else {                                          // the last, partial k-tile
          for (int kk = 0; kk < n_mma; ++kk) {
            const int atom = FMT == 1 ? kk : kk / 2;
            const uint32_t sf_id = FMT == 1 ? 0u : uint32_t(kk & 1) * 2u;
            tc_mma<FMT>(tmem + ACC_COL, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk),
                        idesc(FMT, BN, BM, sf_id, sf_id), (sfbase + 4 * atom) | (sf_id << 30),
                        (sfbase + SFB_OFF + 8 * atom) | (sf_id << 30), (kt > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(&empty[s]);
        tc_commit(&sf_empty[buf]);
        if (kt == nkt - 1) tc_commit(acc_full);
        if (++buf == NSF) { buf = 0; sph ^= 1; }
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      acc_ph ^= 1;
    }
  } else if (warp >= 8) {
    // ------------------------------------------- scale factors -> TMEM --
    // Lane l of warp q copies row l of every scale atom of the stage (16 bytes
    // = the scales of rows l, l+32, l+64, l+96) into TMEM lane 32q + l: the
    // same replicated layout tcgen05.cp .32x128b.warpx4 produces.
    const int q = warp & 3;
    int s = 0, buf = 0;
    uint32_t ph = 0;
    uint32_t sph = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
      for (int64_t kt = 0; kt < nkt; ++kt) {
        const bool a = mbar_wait(&sf_empty[buf], sph ^ 1u, abort_flag, p.status);
        const bool b = a && mbar_wait(&full[s], ph, abort_flag, p.status);
        if (__any_sync(0xFFFFFFFFu, !b)) { ok = false; break; }
        tc_fence_after();
        uint32_t va[16], vb[32];
        const uint8_t* sa = sSFA + s * SFA_BYTES + lane * 16;
        const uint8_t* sb = sSFB + s * SFB_BYTES + lane * 16;
#pragma unroll
        for (int at = 0; at < 4; ++at) {
          const uint4 x = *reinterpret_cast<const uint4*>(sa + at * 512);
          va[4 * at] = x.x; va[4 * at + 1] = x.y; va[4 * at + 2] = x.z; va[4 * at + 3] = x.w;
#pragma unroll
          for (int rb = 0; rb < 2; ++rb) {
            const uint4 y = *reinterpret_cast<const uint4*>(sb + (rb * 4 + at) * 512);
            const int o = 8 * at + 4 * rb;
            vb[o] = y.x; vb[o + 1] = y.y; vb[o + 2] = y.z; vb[o + 3] = y.w;
          }
        }
        const uint32_t base = tmem + (uint32_t(q * 32) << 16) + SF_COL + SF_BUF_COLS * uint32_t(buf);
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(base),
            "r"(va[0]), "r"(va[1]), "r"(va[2]), "r"(va[3]), "r"(va[4]), "r"(va[5]), "r"(va[6]), "r"(va[7]), "r"(va[8]),
            "r"(va[9]), "r"(va[10]), "r"(va[11]), "r"(va[12]), "r"(va[13]), "r"(va[14]), "r"(va[15]));
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
            "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(base + SFB_OFF),
            "r"(vb[0]), "r"(vb[1]), "r"(vb[2]), "r"(vb[3]), "r"(vb[4]), "r"(vb[5]), "r"(vb[6]), "r"(vb[7]), "r"(vb[8]),
            "r"(vb[9]), "r"(vb[10]), "r"(vb[11]), "r"(vb[12]), "r"(vb[13]), "r"(vb[14]), "r"(vb[15]), "r"(vb[16]),
            "r"(vb[17]), "r"(vb[18]), "r"(vb[19]), "r"(vb[20]), "r"(vb[21]), "r"(vb[22]), "r"(vb[23]), "r"(vb[24]),
            "r"(vb[25]), "r"(vb[26]), "r"(vb[27]), "r"(vb[28]), "r"(vb[29]), "r"(vb[30]), "r"(vb[31]));
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        mbar_arrive(&sf_full[buf]);
        if (++buf == NSF) { buf = 0; sph ^= 1; }
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------------------------------- epilogue --
    // TMEM -> registers -> (scale, Quartet mask + H32^-1) -> 128-byte-swizzled
    // staging in shared memory -> TMA store.  The accumulator is released as
    // soon as its last columns are in registers, so the next tile's MMAs
    // overlap the stores.
    constexpr int CW = OUT == OUT_F32 ? 32 : 64;       // columns per 128-byte staged row
    const int q = warp & 3, tid = threadIdx.x - 128, rl = q * 32 + lane;
    uint32_t acc_ph = 0;
    int chunk = 0;
    const float tscale = __fmul_rn(*p.ta, *p.tb);
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
      int64_t mb, nb;
      tile_coords(t, nm, nn, mb, nb);
      const bool got = mbar_wait(acc_full, acc_ph, abort_flag, p.status);
      if (epi_any(!got)) break;                         // uniform decision across the 4 warps
      acc_ph ^= 1;
      tc_fence_after();
      const int64_t row = mb * BM + rl;
      for (int c = 0; c < BN / CW; ++c) {
        float v[CW];
#pragma unroll
        for (int i = 0; i < CW / 32; ++i)
          tmem_ld32(tmem + ACC_COL + (uint32_t(q * 32) << 16) + c * CW + 32 * i, v + 32 * i);
        if (c == BN / CW - 1) {                         // accumulator fully read: release it
          tc_fence_before();
          mbar_arrive(acc_empty);
        }
        const int64_t col0 = nb * BN + c * CW;
#pragma unroll
        for (int j = 0; j < CW; ++j) v[j] = v[j] * tscale;
        if (EPI == 1) {
#pragma unroll
          for (int hb = 0; hb < CW / 32; ++hb) {
            float* u = v + 32 * hb;
            const int64_t cb = col0 + 32 * hb;
            if (p.mask && row < p.M && cb < p.N) {
              const uint32_t mw = *reinterpret_cast<const uint32_t*>(p.mask + row * (p.N >> 3) + (cb >> 3));
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if ((mw >> j) & 1u) u[j] = 0.0f;
            }
#pragma unroll
            for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                if (i & h) continue;
                float a = u[i], b = u[i + h];
                u[i] = a + b;
                u[i + h] = a - b;
              }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) u[j] *= 0.176776695296636881f;
          }
        }
        uint32_t wds[32];
        if (OUT == OUT_F32) {
#pragma unroll
          for (int j = 0; j < 32; ++j) wds[j] = __float_as_uint(v[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            wds[j] = *reinterpret_cast<uint32_t*>(&h2);
          }
        }
        uint8_t* stg = sStage + (chunk & 1) * STG_BYTES;
        if (tid == 0) bulk_wait_read1();                // the store that last used this buffer has read it
        epi_bar();
#pragma unroll
        for (int j = 0; j < 8; ++j)                     // 16-byte chunk j of row rl, 128B-swizzled
          *reinterpret_cast<uint4*>(stg + rl * 128 + ((j ^ (rl & 7)) << 4)) =
              make_uint4(wds[4 * j], wds[4 * j + 1], wds[4 * j + 2], wds[4 * j + 3]);
        fence_proxy_async();
        epi_bar();
        if (tid == 0) {
          tma_store_2d(&map_d, stg, int(col0), int(mb * BM));
          bulk_commit();
        }
        ++chunk;
      }
    }
    if (tid == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

// ------------------------------------------------- CTA-pair (2-SM) kernel --
// The same GEMM on 256 x 256 output tiles computed by a cluster of two CTAs
// with cta_group::2 MMAs: CTA r of the pair loads rows r*128.. of the tile's A
// rows and of its B rows, the leader (rank 0) issues MMAs with M = 256 that
// read both CTAs' shared memory, and each CTA keeps its 128 x 256 half of the
// accumulator in its own tensor memory.  Each CTA thus moves half the B
// bytes per MMA of the one-CTA kernel, which buys two more pipeline stages.
//   operands: both CTAs' TMA loads (warp 0) complete on the leader's
//             full[s] (expected bytes set by the leader's producer);
//   scales:   each CTA copies its own scale atoms (its 128 A rows, all 256 B
//             rows; warp 3) into its sf_ld[s], and its stagers write them
//             into TMEM scale buffer s, then arrive on the leader's full[s]
//             (one producer arrival + 8 stager-warp arrivals + the bytes);
//   releases: the leader's commits arrive on empty[s] and acc_full in both
//             CTAs (tcgen05.commit multicast);
//   epilogue: each CTA drains its half and arrives on the leader's acc_empty.
// The leader's MMA thread thus waits on one barrier and commits one release
// per k-tile: its own instruction stream, not the tensor pipe, sets the pace
// when it has more to do per k-tile.
namespace pair {

constexpr int STAGES = 5;
constexpr int A_BYTES = 128 * 128;                   // this CTA's 128 A rows x 128 bytes
constexpr int B_BYTES = 128 * 128;                   // this CTA's 128 B rows
constexpr int SFA_BYTES = 4 * 512;
constexpr int SFB_BYTES = 8 * 512;                   // both 128-row blocks of the tile's B
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 2 * STG_BYTES + 1024 + 256;
// 16 warps: producer, MMA issuer, TMEM allocator, spare | 4 scale stagers |
// 8 epilogue warps (two per TMEM lane quadrant, 128 columns each).  The
// block launches with 128 registers a thread (65536); the first two
// warpgroups give registers back so the epilogue can hold 128 accumulator
// columns per thread: 128 x (56 + 80 + 184 + 184) = 64512 <= 65536.
constexpr int PTHREADS = 512;
constexpr int REG_CTRL = 56, REG_STAGE = 80, REG_EPI = 184;
static_assert(128 * (REG_CTRL + REG_STAGE + 2 * REG_EPI) <= 65536, "register split of the CTA-pair kernel");
static_assert(SMEM_BYTES <= 232448, "shared memory of the CTA-pair kernel");
static_assert(SF_COL + STAGES * SF_BUF_COLS <= TMEM_COLS, "one scale TMEM buffer per stage");

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared::cluster address of the same object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// Arrive on a barrier of either CTA of the pair (default .release.cta
// semantics: the data it orders is tensor-memory state, ordered by the
// tcgen05 fences around the arrive and the wait).
__device__ __forceinline__ void arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool try_c(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: false and the abort flag raised when the limit is hit.
__device__ __forceinline__ bool wait_c(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* status) {
  if (try_c(b, parity)) return true;
  const unsigned long long t0 = clock64();
  while (true) {
    if (try_c(b, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > WAIT_LIMIT) {
      *abort_flag = 1;
      flag_status(status, ST_TIMEOUT);
      return false;
    }
  }
}

// TMA tile load whose completion is counted on the leader CTA's barrier (the
// barrier address with the peer bit cleared).
__device__ __forceinline__ void tma_load_pair(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar) & 0xFEFFFFFFu)
      : "memory");
}

__device__ __forceinline__ void commit_both(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void commit_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Named barrier of the four epilogue warps that cover one 128-column half.
__device__ __forceinline__ void half_bar(int h) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + h) : "memory");
}
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

template <int FMT>
__device__ __forceinline__ void mma_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                         uint32_t sfb, uint32_t acc) {
  if (FMT == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
  }
}

}  // namespace pair

template <int FMT, int NK, bool PAIR>
__device__ __forceinline__ void mma_ktile(uint32_t acc, uint64_t ad, uint64_t bd, uint32_t sfbase, uint32_t idesc0,
                                          bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < NK; ++kk) {
    const int atom = FMT == 1 ? kk : kk / 2;
    const uint32_t sf_id = FMT == 1 ? 0u : uint32_t(kk & 1) * 2u;
    const uint32_t id = idesc0 | (sf_id << 4) | (sf_id << 29);
    const uint32_t sfa = (sfbase + 4 * atom) | (sf_id << 30), sfb = (sfbase + SFB_OFF + 8 * atom) | (sf_id << 30);
    const uint32_t c = (kk > 0 || accumulate) ? 1u : 0u;
    if (PAIR) pair::mma_pair<FMT>(acc, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), id, sfa, sfb, c);
    else tc_mma<FMT>(acc, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), id, sfa, sfb, c);
  }
}

namespace pair {

// Pair tile order.  raster > 0: groups of `raster` 256-row blocks sweep all
// 256-column blocks (each B tile is fetched once per group and shared by the
// group's tiles of one wave); raster < 0: groups of -raster column blocks
// sweep all row blocks (the same with A and B exchanged).
__device__ __forceinline__ void tile_coords2(int64_t t, int64_t nm, int64_t nn, int raster, int64_t& mb,
                                             int64_t& nb) {
  if (raster < 0) {
    const int64_t G = -raster;
    const int64_t per_group = G * nm;
    const int64_t g = t / per_group, r = t % per_group;
    const int64_t gn = nn - g * G < G ? nn - g * G : G;
    nb = g * G + r % gn;
    mb = r / gn;
    return;
  }
  const int64_t G = raster;
  const int64_t per_group = G * nn;
  const int64_t g = t / per_group, r = t % per_group;
  const int64_t gm = nm - g * G < G ? nm - g * G : G;
  mb = g * G + r % gm;
  nb = r / gm;
}

template <int FMT, int OUT, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PTHREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_d, const __grid_constant__ CUtensorMap map_sfa,
                const __grid_constant__ CUtensorMap map_sfb, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sSFA = sB + STAGES * B_BYTES;
  uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;
  uint8_t* sStage = sSFB + STAGES * SFB_BYTES;
  // Stage s owns an operand slot, a scale slot and scale TMEM buffer s.
  uint64_t* full = reinterpret_cast<uint64_t*>(sStage + 2 * STG_BYTES);   // leader: operand bytes of both CTAs
                                                                            // + 4 stager warps x 2 CTAs
  uint64_t* empty = full + STAGES;                                          // both: stage consumed by the MMAs
  uint64_t* sf_ld = empty + STAGES;                                         // both: this CTA's scale atoms landed
  uint64_t* sf_free = sf_ld + STAGES;                                       // both: the stagers have read them
  uint64_t* acc_full = sf_free + STAGES;                                    // both
  uint64_t* acc_empty = acc_full + 1;                                       // leader: 4 warps x 2 CTAs
  uint64_t* drain = acc_empty + 1;                                          // leader: MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool leader = rank == 0;
  const int64_t nm = (p.M + 255) / 256, nn = (p.N + BN - 1) / BN, ntiles = nm * nn;
  const int64_t nkt = (p.K + BK - 1) / BK;
  const int64_t pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  constexpr int G = FMT == 1 ? 16 : 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1 + 8);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ld[s], 1);
      mbar_init(&sf_free[s], 4);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 16);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();                                   // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // warpgroup of this warp, warp-uniform for the compiler
  const int wg = __shfl_sync(0xFFFFFFFFu, int(threadIdx.x) >> 7, 0);
  // the leader's barriers that both CTAs arrive on
  const uint32_t acc_empty_l = mapa(acc_empty, 0);

  if (wg == 0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_CTRL));
  if ((warp == 0 || warp == 3) && lane == 0) {
    // --------------------------------------------- producers (2 threads) --
    // Warp 0 loads the operand tiles (TMA, completing on the leader's
    // full[s]), warp 3 this CTA's scale atoms (3-D TMA, on its own
    // sf_ld[s]): one thread issuing every copy of a k-tile is itself the
    // bottleneck at this rate.  Both walk the same stages; the operands wait
    // for the MMAs to release a stage, the scale atoms only for the stagers
    // to have read its slot, so their copies run up to a ring ahead.
    const bool operands = warp == 0;
    int s = 0;
    uint32_t ph = 0;
    const int64_t nrb_a = (p.M + 127) / 128, nrb_b = (p.N + 127) / 128;
    const int nk = int(nkt);
    int* const st = p.status;
    for (int64_t t = pair_id; t < ntiles && !*abort_flag; t += npairs) {
      int64_t mb, nb;
      tile_coords2(t, nm, nn, p.raster, mb, nb);
      const int64_t ra = mb * 2 + rank, rb = nb * 2 + rank;          // this CTA's 128-row blocks
      // 128-row halves that exist (a half entirely past M or N is not loaded)
      const int a_halves = (mb * 2 + 1 < nrb_a) ? 2 : 1, b_halves = (nb * 2 + 1 < nrb_b) ? 2 : 1;
      const bool load_a = ra < nrb_a, load_b = rb < nrb_b;
      const uint32_t op_bytes = uint32_t((a_halves + b_halves) * A_BYTES);
      for (int kt = 0; kt < nk; ++kt) {
        // operands wait for the MMAs to release the stage; scale atoms only for
        // the stagers to have read the slot (they run up to a ring ahead)
        if (!wait_c(operands ? &empty[s] : &sf_free[s], ph ^ 1, abort_flag, st)) break;
        if (operands) {
          if (leader) mbar_expect_tx(&full[s], op_bytes);
          if (load_a) tma_load_pair(sA + s * A_BYTES, &map_a, kt * (BK / 2), int(ra * 128), &full[s]);
          if (load_b) tma_load_pair(sB + s * B_BYTES, &map_b, kt * (BK / 2), int(rb * 128), &full[s]);
        } else {
          // Scale atoms through 3-D views {128 words, atom, 128-row block} of
          // the tensor-core scale layout: 4 atoms of this CTA's A rows, and
          // 4 atoms x both 128-row blocks of the tile's B rows, in one copy
          // each (atoms past the last, or a B block past N, read as zeros).
          const int atom0 = kt * (BK / G / 4);
          mbar_expect_tx(&sf_ld[s], uint32_t(load_a ? SFA_BYTES : 0) + uint32_t(SFB_BYTES));
          if (load_a) tma_load_3d(sSFA + s * SFA_BYTES, &map_sfa, 0, atom0, int(ra), &sf_ld[s]);
          tma_load_3d(sSFB + s * SFB_BYTES, &map_sfb, 0, atom0, int(nb * 2), &sf_ld[s]);
        }
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
    }
    if (*abort_flag) {                               // let copies already issued land before teardown
      const unsigned long long t0 = clock64();
      while (clock64() - t0 < 4000000ull) {}
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // --------------------------------------------------------- MMA issue --
    // One thread issues every MMA, and its own scalar work per loop trip
    // (counters, descriptors, parameter loads) costs about as much as the
    // four MMAs of a k-tile take on the tensor pipe.  So the loop is lean: all
    // bases are in registers, counters are 32-bit, and each trip takes two
    // k-tiles (each waited for, issued and released on its own).
    int s = 0;
    uint32_t ph = 0, acc_ph = 0;
    bool ok = true, issued = false;
    const int nk = int(nkt);
    const int last_mma = int((p.K - int64_t(nk - 1) * BK) / 64);   // MMAs of the last k-tile
    int* const st = p.status;
    const uint64_t ad0 = desc_sw128(smem_u32(sA)), bd0 = desc_sw128(smem_u32(sB));
    const uint32_t id0 = idesc(FMT, BN, 256, 0, 0), acc_t = tmem + ACC_COL, sf0 = tmem + SF_COL;
    // Waits for stage s (operands of both CTAs and the scales in TMEM),
    // issues k-tile kt from it and releases it; false when the wait gave up.
    auto ktile = [&](int kt) -> bool {
      if (!wait_c(&full[s], ph, abort_flag, st)) return false;
      tc_fence_after();
      const uint64_t ad = ad0 + uint64_t(s * (A_BYTES >> 4)), bd = bd0 + uint64_t(s * (B_BYTES >> 4));
      const uint32_t sfbase = sf0 + SF_BUF_COLS * uint32_t(s);
      if (kt + 1 < nk || last_mma == BK / 64) {
        mma_ktile<FMT, BK / 64, true>(acc_t, ad, bd, sfbase, id0, kt > 0);
      } else {                                        // the last, partial k-tile
        for (int kk = 0; kk < last_mma; ++kk) {
          const int atom = FMT == 1 ? kk : kk / 2;
          const uint32_t sf_id = FMT == 1 ? 0u : uint32_t(kk & 1) * 2u;
          mma_pair<FMT>(acc_t, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), idesc(FMT, BN, 256, sf_id, sf_id),
                        (sfbase + 4 * atom) | (sf_id << 30), (sfbase + SFB_OFF + 8 * atom) | (sf_id << 30),
                        (kt > 0 || kk > 0) ? 1u : 0u);
        }
      }
      commit_both(&empty[s]);
      if (kt == nk - 1) commit_both(acc_full);
      if (++s == STAGES) { s = 0; ph ^= 1; }
      return true;
    };
    for (int64_t t = pair_id; ok && t < ntiles && !*abort_flag; t += npairs) {
      if (!wait_c(acc_empty, acc_ph ^ 1, abort_flag, st)) break;
      tc_fence_after();
      issued = true;
      for (int kt = 0; kt < nk; kt += 2) {
        if (!ktile(kt)) { ok = false; break; }
        if (kt + 1 < nk && !ktile(kt + 1)) { ok = false; break; }
      }
      acc_ph ^= 1;
    }
    if (issued) {                                    // every MMA retired before teardown
      commit_local(drain);                           // (bounded, and also after an abort)
      const unsigned long long t0 = clock64();
      while (!try_c(drain, 0) && clock64() - t0 < WAIT_LIMIT) {}
    }
  }
  } else if (wg == 1) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_STAGE));
    // ------------------------------------------- scale factors -> TMEM --
    // Each stager warp reads stage s's scale atoms once they have landed,
    // frees the slot for the next round's copies (sf_free), waits for the
    // MMAs that last read scale TMEM buffer s to retire (empty), writes the
    // buffer and arrives on the leader's full[s].
    const int q = warp & 3;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    const uint32_t full_l = mapa(full, 0);
    for (int64_t t = pair_id; ok && t < ntiles; t += npairs) {
      for (int64_t kt = 0; kt < nkt; ++kt) {
        const bool b = wait_c(&sf_ld[s], ph, abort_flag, p.status);
        if (__any_sync(0xFFFFFFFFu, !b)) { ok = false; break; }
        tc_fence_after();
        uint32_t va[16], vb[32];
        const uint8_t* sa = sSFA + s * SFA_BYTES + lane * 16;
        const uint8_t* sb = sSFB + s * SFB_BYTES + lane * 16;
#pragma unroll
        for (int at = 0; at < 4; ++at) {
          const uint4 x = *reinterpret_cast<const uint4*>(sa + at * 512);
          va[4 * at] = x.x; va[4 * at + 1] = x.y; va[4 * at + 2] = x.z; va[4 * at + 3] = x.w;
#pragma unroll
          for (int rbk = 0; rbk < 2; ++rbk) {
            const uint4 y = *reinterpret_cast<const uint4*>(sb + (rbk * 4 + at) * 512);
            const int o = 8 * at + 4 * rbk;
            vb[o] = y.x; vb[o + 1] = y.y; vb[o + 2] = y.z; vb[o + 3] = y.w;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_free[s]);     // the slot may be refilled
        // scale TMEM buffer s is free once the MMAs of its previous round retired
        const bool e = wait_c(&empty[s], ph ^ 1, abort_flag, p.status);
        if (__any_sync(0xFFFFFFFFu, !e)) { ok = false; break; }
        tc_fence_after();
        const uint32_t base = tmem + (uint32_t(q * 32) << 16) + SF_COL + SF_BUF_COLS * uint32_t(s);
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(base),
            "r"(va[0]), "r"(va[1]), "r"(va[2]), "r"(va[3]), "r"(va[4]), "r"(va[5]), "r"(va[6]), "r"(va[7]), "r"(va[8]),
            "r"(va[9]), "r"(va[10]), "r"(va[11]), "r"(va[12]), "r"(va[13]), "r"(va[14]), "r"(va[15]));
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
            "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(base + SFB_OFF),
            "r"(vb[0]), "r"(vb[1]), "r"(vb[2]), "r"(vb[3]), "r"(vb[4]), "r"(vb[5]), "r"(vb[6]), "r"(vb[7]), "r"(vb[8]),
            "r"(vb[9]), "r"(vb[10]), "r"(vb[11]), "r"(vb[12]), "r"(vb[13]), "r"(vb[14]), "r"(vb[15]), "r"(vb[16]),
            "r"(vb[17]), "r"(vb[18]), "r"(vb[19]), "r"(vb[20]), "r"(vb[21]), "r"(vb[22]), "r"(vb[23]), "r"(vb[24]),
            "r"(vb[25]), "r"(vb[26]), "r"(vb[27]), "r"(vb[28]), "r"(vb[29]), "r"(vb[30]), "r"(vb[31]));
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_cluster(full_l + uint32_t(s) * 8u);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_EPI));
    // ---------------------------------------------------------- epilogue --
    // warp 8 + 4h + q holds TMEM lane quadrant q (rows 32q..32q+31 of this
    // CTA's half) and columns 128h .. 128h+127: all of them are read into
    // registers and the accumulator is released (on the leader's
    // acc_empty) before any store, so the next tile's MMAs overlap the
    // stores; then the four warps of half h store 32-column (fp32) or
    // 64-column (bf16) chunks through the half's 128-byte-swizzled staging
    // buffer with TMA stores.
    constexpr int CW = OUT == OUT_F32 ? 32 : 64;
    const int q = warp & 3, h = (warp - 8) >> 2, rl = q * 32 + lane;
    const bool storer = q == 0 && lane == 0;        // one thread per half issues its stores
    uint8_t* stg = sStage + h * STG_BYTES;
    uint32_t acc_ph = 0;
    const float tscale = __fmul_rn(*p.ta, *p.tb);
    for (int64_t t = pair_id; t < ntiles; t += npairs) {
      int64_t mb, nb;
      tile_coords2(t, nm, nn, p.raster, mb, nb);
      const bool got = wait_c(acc_full, acc_ph, abort_flag, p.status);
      uint32_t bad;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
          "bar.red.or.pred q, 3, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(bad)
          : "r"(uint32_t(!got))
          : "memory");
      if (bad) break;                                // uniform across the 8 epilogue warps
      acc_ph ^= 1;
      tc_fence_after();
      float v[128];
#pragma unroll
      for (int i = 0; i < 4; ++i) tmem_ld32_async(tmem + ACC_COL + (uint32_t(q * 32) << 16) + 128 * h + 32 * i, v + 32 * i);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_cluster(acc_empty_l);
      const int64_t row0 = mb * 256 + int64_t(rank) * 128, row = row0 + rl;
#pragma unroll
      for (int j = 0; j < 128; ++j) v[j] = v[j] * tscale;
      if (EPI == 1) {
#pragma unroll
        for (int hb = 0; hb < 4; ++hb) {
          float* u = v + 32 * hb;
          const int64_t cb = nb * BN + 128 * h + 32 * hb;
          if (p.mask && row < p.M && cb < p.N) {
            const uint32_t mw = *reinterpret_cast<const uint32_t*>(p.mask + row * (p.N >> 3) + (cb >> 3));
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if ((mw >> j) & 1u) u[j] = 0.0f;
          }
#pragma unroll
          for (int hh = 1; hh < 32; hh <<= 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (i & hh) continue;
              float a = u[i], b = u[i + hh];
              u[i] = a + b;
              u[i + hh] = a - b;
            }
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] *= 0.176776695296636881f;
        }
      }
#pragma unroll
      for (int c = 0; c < 128 / CW; ++c) {
        uint32_t wds[32];
        if (OUT == OUT_F32) {
#pragma unroll
          for (int j = 0; j < 32; ++j) wds[j] = __float_as_uint(v[CW * c + j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(v[CW * c + 2 * j], v[CW * c + 2 * j + 1]);
            wds[j] = *reinterpret_cast<uint32_t*>(&h2);
          }
        }
        if (storer) bulk_wait_read0();               // the previous store has read the buffer
        half_bar(h);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(stg + rl * 128 + ((j ^ (rl & 7)) << 4)) =
              make_uint4(wds[4 * j], wds[4 * j + 1], wds[4 * j + 2], wds[4 * j + 3]);
        fence_proxy_async();
        half_bar(h);
        if (storer && row0 < p.M) {
          tma_store_2d(&map_d, stg, int(nb * BN + 128 * h + CW * c), int(row0));
          bulk_commit();
        }
      }
    }
    if (storer) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();                                   // no arrivals or MMAs into the peer remain
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

}  // namespace pair

// ------------------------------------------------------------ host side --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Codes of a rows x K tensor as a 2-D uint8 tensor (K/2 bytes per row), box
// 128 bytes x box_rows, 128-byte swizzle, zero fill outside.
static bool make_map(CUtensorMap* m, const void* codes, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cuuint64_t(K / 2), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(K / 2)};
  cuuint32_t box[2] = {128, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output D (M x N, fp32 or bf16) for the epilogue's TMA stores: box of 128
// bytes x 128 rows, 128-byte swizzle (the staging layout); out-of-range rows
// and columns of a tile are not written.
static bool make_map_d(CUtensorMap* m, void* D, int64_t M, int64_t N, int out_dtype) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int es = out_dtype ? 2 : 4;
  cuuint64_t dims[2] = {cuuint64_t(N), cuuint64_t(M)};
  cuuint64_t strides[1] = {cuuint64_t(N) * cuuint64_t(es)};
  cuuint32_t box[2] = {cuuint32_t(128 / es), cuuint32_t(BM)};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, out_dtype ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, D, dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor-core scale layout of a rows x groups scale matrix as a 3-D tensor
// of 32-bit words {128 words of an atom, nkb atoms of a 128-row block, row
// blocks}; box {128, 4, box_blocks} (4 atoms: one k-tile of 256 elements for
// NVFP4, two for MXFP4); reads past the end return zeros.
static bool make_map_sf(CUtensorMap* m, const uint8_t* swz, int64_t rows, int64_t nkb, int box_blocks) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, cuuint64_t(nkb), cuuint64_t((rows + 127) / 128)};
  cuuint64_t strides[2] = {512, cuuint64_t(nkb) * 512};
  cuuint32_t box[3] = {128, 4, cuuint32_t(box_blocks)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t*>(swz), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, int OUT, int EPI>
static cudaError_t launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& md, const Params& p,
                          cudaStream_t s) {
  auto kern = k_gemm<FMT, OUT, EPI>;
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);   // idempotent: racing threads set the same value
  }
  int64_t tiles = ((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
  int grid = int(tiles < num_sms() ? tiles : num_sms());
  kern<<<grid, THREADS, SMEM_BYTES, s>>>(ma, mb, md, p);
  count_launch();
  return cudaGetLastError();
}

// CTA-pair launch: one 2-CTA cluster per resident pair of SMs (as many as
// the device co-schedules), grid-stride over the 256 x 256 tiles.
template <int FMT, int OUT, int EPI>
static cudaError_t launch_pair(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& md,
                               const Params& p, cudaStream_t s) {
  CUtensorMap msa, msb;
  if (!make_map_sf(&msa, p.sfa, p.M, p.nkb, 1) || !make_map_sf(&msb, p.sfb, p.N, p.nkb, 2)) return cudaErrorInvalidValue;
  auto kern = pair::k_gemm_pair<FMT, OUT, EPI>;
  static std::atomic<int> max_clusters[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int mc = max_clusters[dev].load(std::memory_order_acquire);
  if (mc == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pair::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * unsigned(num_sms() / 2));
    cfg.blockDim = dim3(pair::PTHREADS);
    cfg.dynamicSmemBytes = pair::SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = num_sms() / 2;
    }
    mc = n;
    max_clusters[dev].store(mc, std::memory_order_release);   // idempotent: racing threads store the same value
  }
  const int64_t tiles = ((p.M + 255) / 256) * ((p.N + BN - 1) / BN);
  const int64_t pairs = tiles < mc ? tiles : mc;
  kern<<<unsigned(2 * pairs), pair::PTHREADS, pair::SMEM_BYTES, s>>>(ma, mb, md, msa, msb, p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace gemm
}  // namespace fp4

using namespace fp4;

extern "C" int fp4_gemm(const fp4_qtensor* A, const fp4_qtensor* B, void* D, int32_t out_dtype,
                        const uint8_t* epi_mask, int32_t epi_inverse_had, fp4_stream_t stream) {
  if (!A || !B) return FP4_ERR_INVALID_ARG;
  if (A->fmt != B->fmt || (A->fmt != FP4_MXFP4 && A->fmt != FP4_NVFP4)) return FP4_ERR_INVALID_ARG;
  if (out_dtype != 0 && out_dtype != 1) return FP4_ERR_INVALID_ARG;
  if (epi_inverse_had != 0 && epi_inverse_had != 32) return FP4_ERR_UNSUPPORTED;
  if (epi_mask && !epi_inverse_had) return FP4_ERR_UNSUPPORTED;
  const int64_t M = A->rows, N = B->rows, K = A->cols;
  if (M < 0 || N < 0 || K < 0 || B->cols != K) return FP4_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FP4_OK;
  if (K % 64 || N % 8) return FP4_ERR_INVALID_ARG;
  if (epi_inverse_had && N % 32) return FP4_ERR_INVALID_ARG;
  if (!A->codes || !B->codes || !A->scales_swz || !B->scales_swz || !A->tensor_scale ||
      !B->tensor_scale || !D)
    return FP4_ERR_INVALID_ARG;
  auto al = [](const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (!al(A->codes, 16) || !al(B->codes, 16) || !al(A->scales_swz, 16) || !al(B->scales_swz, 16) ||
      !al(D, 16) || (epi_mask && !al(epi_mask, 4)))
    return FP4_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) {
    size_t bytes = size_t(M) * size_t(N) * (out_dtype ? 2 : 4);
    return cudaMemsetAsync(D, 0, bytes, s) == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
  }
  // Two-CTA (cta_group::2) kernel unless M fits one 128-row block, where the
  // second CTA of every pair would have no rows.  FP4_GEMM_PAIR=0 in the
  // environment selects the one-CTA kernel for every shape (read per call).
  const char* pair_env = getenv("FP4_GEMM_PAIR");
  const bool use_pair = M > gemm::BM && !(pair_env && pair_env[0] == '0');
  CUtensorMap ma, mb, md;
  if (!gemm::make_map(&ma, A->codes, M, K, gemm::BM) ||
      !gemm::make_map(&mb, B->codes, N, K, use_pair ? 128 : gemm::BN) || !gemm::make_map_d(&md, D, M, N, out_dtype))
    return FP4_ERR_CUDA;
  gemm::Params p{};
  p.M = M; p.N = N; p.K = K;
  p.sfa = A->scales_swz; p.sfb = B->scales_swz;
  p.nkb = (K / (A->fmt == FP4_NVFP4 ? 16 : 32) + 3) / 4;
  p.ta = A->tensor_scale; p.tb = B->tensor_scale;
  p.D = D; p.mask = epi_mask; p.status = status_ptr();
  // Tile order of the pair kernel (measured on the Llama-shaped layer set):
  // with at least as many rows as columns, groups of 8 column blocks sweep
  // the rows; otherwise groups of 16 row blocks sweep the columns.
  p.raster = M >= N ? -8 : 16;
  cudaError_t e;
  const bool nv = A->fmt == FP4_NVFP4, bf = out_dtype == 1, epi = epi_inverse_had == 32;
#define FP4_GEMM_LAUNCH(F, O, E) \
  (use_pair ? gemm::launch_pair<F, O, E>(ma, mb, md, p, s) : gemm::launch<F, O, E>(ma, mb, md, p, s))
  if (nv) {
    if (bf) e = epi ? FP4_GEMM_LAUNCH(1, 1, 1) : FP4_GEMM_LAUNCH(1, 1, 0);
    else e = epi ? FP4_GEMM_LAUNCH(1, 0, 1) : FP4_GEMM_LAUNCH(1, 0, 0);
  } else {
    if (bf) e = epi ? FP4_GEMM_LAUNCH(0, 1, 1) : FP4_GEMM_LAUNCH(0, 1, 0);
    else e = epi ? FP4_GEMM_LAUNCH(0, 0, 1) : FP4_GEMM_LAUNCH(0, 0, 0);
  }
#undef FP4_GEMM_LAUNCH
  return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}
