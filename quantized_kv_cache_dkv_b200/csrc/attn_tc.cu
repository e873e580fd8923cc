// Bidirectional block attention over the low-bit cache on the 5th-generation
// tensor cores (tcgen05 + tensor memory).  A query group (query heads per
// kv-head x block tokens, 32..256 rows) is processed in row blocks of at most
// 128 rows, each padded with zero queries to the M = 128 MMA shape.  The
// scores and the weighted sum read the packed codes themselves, at each
// denoising step (MaskAhead / Q-MaskAhead abstract: Q-MaskAhead attends over
// the low-bit cache without a dequantized copy).
//
// CTA = (unit, token split, row block), one CTA per SM, 28 warps (seven
// warpgroups; setmaxnreg: softmax 96 registers, producers 64, control 56):
//   warps 0-7   softmax, two warpgroups: warpgroup h takes the 128-token
//               tiles j = h (mod 2); thread = query row = TMEM lane, all 128
//               columns.  Loads its half of Q into TMEM; per tile: the row
//               max of S (pass 1), the reference max handed over from the
//               previous tile through shared memory (raised only when the
//               tile max exceeds it by more than 8 in log2 units, so P <= 2^8),
//               P = 2^(s*scale - ref) as fp16 pairs written over the first 64
//               columns of its S buffer (pass 2), O rescaled in TMEM when the
//               reference rose; at the end the two warpgroups' row sums are
//               merged and each writes half of the output / split partial
//   warps 8-15  K producers: dequantize 128-token K tiles into shared memory
//               (channel rows, tokens contiguous: MN-major, 128-byte swizzle);
//               two warps per SM sub-partition, half a tile each
//   warps 16-23 V producers: dequantize V tiles (token rows, channels
//               contiguous: MN-major, 128-byte swizzle), half a tile each
//   warp 25     allocates TMEM; one lane issues the MMAs:
//               S_j = Q K_j^T (A = Q from TMEM), O += P_j V_j (A = P from TMEM)
//   warp 26     one lane streams each tile's packed K/V codes and fp16
//               (scale, zero) pairs -- four contiguous ranges of the cache --
//               and the tile's slice of the protected-K side table into a
//               3-stage shared-memory ring with 1-D bulk copies
//               (cp.async.bulk, completion counted on an mbarrier), so HBM
//               latency overlaps the dequantization and the MMAs
// Tensor memory (512 columns x 128 lanes x 32 bit): O [0,128), S0 [128,256),
// S1 [256,384), Q [384,448).  P_j (fp16 pairs) overwrites the first 64
// columns of S_(j mod 2) once the scores are read; the PV MMAs take their A
// operand there.
// Hand-offs are mbarriers; MMA completion arrives through tcgen05.commit.
// Every wait is bounded (about one second of %globaltimer): on expiry the
// CTA raises DKV_FLAG_TIMEOUT, all roles leave their loops, the MMA lane waits
// (bounded) for its own MMAs, and TMEM is released before returning.
#include <type_traits>

#include "dequant.cuh"
#include "dkv_internal.cuh"

namespace dkv {
namespace {

// Pipeline trace (trace build, DKV_TRACE, libdkv_trace.so): clock64 stamps of
// CTA 0 of the last launch, per event and tile (first 64 tiles), read with
// dkv_trace_read.  In the normal build the stamps compile to nothing.
#ifdef DKV_TRACE
__device__ unsigned long long g_trace[16][64];
#define DKV_TR(e, j)                                                            \
  do {                                                                          \
    if (blockIdx.x == 0 && (j) < 64) g_trace[e][j] = static_cast<unsigned long long>(clock64()); \
  } while (0)
#else
#define DKV_TR(e, j) \
  do {               \
  } while (0)
#endif
// events: 0 loader issues the tile's copies, 1/2 K producer starts/ends the
// tile, 11/3/4 V producer has its buffer / starts / ends, 5 QK issued, 6
// softmax has the scores, 12 softmax after its first pass or vote, 7 P
// written, 8 PV issue starts, 13 PV issued and committed, 14 QK issued and
// committed, 9 CTA start, 10 CTA end

constexpr int TT = kTcTile;              // tokens per tile
constexpr int kWarps = 28;  // seven warpgroups; warps 26, 27 only complete the last one
constexpr int kThreads = kWarps * 32;
// The MMA lane and the loader sit on sub-partitions 3 and 2: with query
// groups of 32 rows all softmax work lands on sub-partition 0 (TMEM lanes
// 0-31 belong to warps 0 and 4).
constexpr int kMmaWarp = 27;  // sub-partition 3: the MMA issue rate follows its share of issue slots
constexpr int kLoadWarp = 26;
constexpr int kStages = 3;  // ring of packed tiles
constexpr uint32_t kTileBytes = 128 * 128 * 2;
// TMEM columns: O, two score buffers, two P buffers (fp16 pairs).  A score
// buffer is free for the next QK once the softmax has read it, before its P
// is written or multiplied.
constexpr uint32_t kColO = 0, kColS0 = 128, kColS1 = 256, kColP0 = 384, kColP1 = 448,
                   kTmemCols = 512;

// instruction descriptor: D f32, A f16 (K-major), B f16 (MN-major), M = N = 128
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | (0u << 15) | (1u << 16) |
                            ((128u >> 3) << 17) | ((128u >> 4) << 24);

// One ring stage of a tile's packed data, sized for the code widths (byte
// offsets, all multiples of 16): packed K codes (128 tokens x 128 channels x
// KB bits), K (scale, zero) pairs (at most 4 groups x 128 channels), the
// side-table slice of the tile's K groups (header {entries n, first entry
// g0, index base of the staged positions}, positions as an aligned superset,
// the bf16 K rows of the first kProt entries; later ones are read from
// global memory), packed V codes, V (scale, zero) pairs (128 tokens x at
// most 4 groups).
template <int KB, int VB>
struct Stage {
  static constexpr uint32_t kCodesK = KB < 16 ? 2048u * KB : 0u;
  static constexpr uint32_t kCodesV = VB < 16 ? 2048u * VB : 0u;
  static constexpr int kProt = KB >= 16 ? 0 : (KB == 4 && VB == 4 ? 3 : 8);
  static constexpr uint32_t kRKc = 0, kRKsz = kCodesK, kRHdr = kRKsz + (KB < 16 ? 2048u : 0u),
                            kRPos = kRHdr + 16, kRPk = kRPos + 128, kRVc = kRPk + 256u * kProt,
                            kRVsz = kRVc + kCodesV, kBytes = kRVsz + (VB < 16 ? 2048u : 0u);
};
constexpr uint32_t kMaxStageBytes = Stage<4, 4>::kBytes > Stage<2, 4>::kBytes
                                        ? (Stage<4, 4>::kBytes > Stage<4, 2>::kBytes ? Stage<4, 4>::kBytes
                                                                                      : Stage<4, 2>::kBytes)
                                        : Stage<2, 4>::kBytes;
static_assert(Stage<2, 2>::kBytes <= kMaxStageBytes && Stage<2, 16>::kBytes <= kMaxStageBytes &&
                  Stage<4, 16>::kBytes <= kMaxStageBytes && Stage<16, 4>::kBytes <= kMaxStageBytes &&
                  Stage<3, 4>::kBytes <= kMaxStageBytes && Stage<4, 3>::kBytes <= kMaxStageBytes &&
                  Stage<3, 3>::kBytes <= kMaxStageBytes && Stage<3, 16>::kBytes <= kMaxStageBytes &&
                  Stage<16, 3>::kBytes <= kMaxStageBytes,
              "largest ring stage");

struct Smem {
  // offsets into the 1024-byte aligned dynamic shared memory: the two K and
  // the two V tile buffers, Q (the A operand of QK: [128 rows][128
  // channels] fp16, K-major with the 128-byte swizzle, as two halves of 64
  // channels), then the ring
  static constexpr uint32_t kK0 = 0, kK1 = kTileBytes, kV0 = 2 * kTileBytes, kV1 = 3 * kTileBytes;
  static constexpr uint32_t kQ = 4 * kTileBytes;
  static constexpr uint32_t kRing = kQ + kTileBytes;
};
template <int KB, int VB>
struct SmemTail {
  static constexpr uint32_t kBar = Smem::kRing + kStages * Stage<KB, VB>::kBytes;  // 32 mbarriers
  static constexpr uint32_t kRef = kBar + 32 * 8;   // [tile parity][128] reference max per row
  static constexpr uint32_t kLsum = kRef + 1024;    // [warpgroup][128] row sum, then its reference
  static constexpr uint32_t kMisc = kLsum + 2048;   // tmem base, abort flag, then the unit's lengths
  static constexpr uint32_t kBytes = kMisc + 32;
  // plus 1024 bytes of alignment slack
  static_assert(kBytes + 1024 <= 232448, "shared memory per block");
};
enum Bar {
  KFULL = 0, VFULL = 4, VEMPTY = 6, SFULL = 8, PFULL = 10, QREADY = 12, DONE = 13,
  RFULL = 14, REMPTY = 14 + kStages, RREADY = 14 + 2 * kStages, LSUM = RREADY + 2, SFREE = LSUM + 1
};
static_assert(SFREE + 2 <= 32, "barrier slots");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// try_wait suspends the thread until the phase completes or the hint (ns)
// expires, so waiting warps do not take issue slots from working ones
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(200000u)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `parity`; false on abort (unless drain) or after
// a.wait_limit_ns (about 1 s; then the CTA-wide abort flag and the sticky
// timeout flag are set).  `drain` waits that ignore the abort flag are used
// only for the CTA's own copies and MMAs in flight before it releases shared
// and tensor memory.  (`a` is the kernel's __grid_constant__ parameter: its
// fields are read from the parameter bank, not held in registers.)
__device__ bool mbar_wait(uint32_t bar, uint32_t parity, const AttnArgs& a,
                          volatile int* abort_flag, bool drain = false) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 7u) == 7u) {
      if (!drain && *abort_flag) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > a.wait_limit_ns) {
        *abort_flag = 1;
        atomicOr(a.c.status, uint32_t(DKV_FLAG_TIMEOUT));
        return false;
      }
    }
  }
}

// For the producer, loader and MMA loops: the common case -- the phase has
// already completed -- costs one non-blocking test inline; otherwise the
// bounded wait.
__device__ __forceinline__ bool mbar_wait_fast(uint32_t bar, uint32_t parity, const AttnArgs& a,
                                               volatile int* abort_flag) {
  if (mbar_test(bar, parity)) return true;
  return mbar_wait(bar, parity, a, abort_flag);
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// 1-D bulk copy global -> this CTA's own shared memory; completion counted on `bar`
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// shared-memory matrix descriptor, 128-byte swizzle (sm100 descriptor version 1)
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = uint64_t((addr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// Register budgets per warpgroup after setmaxnreg (launch: 72 per thread x
// 896 threads = 64512): softmax rises to 96 (2 x 128 threads), producers drop
// to 64 (512 threads), control to 56 (128 threads): 24576 + 32768 + 7168.
constexpr int kRegSoftmax = 96, kRegProducer = 64, kRegControl = 56;

template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): one instruction for two lanes'
// worth of fma / add / mul, operands as 64-bit register pairs {lo, hi}.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t x, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// D[tmem] (+)= A[tmem] * B[smem]^T
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(accumulate), "r"(kIdesc)
      : "memory");
}

// Eight MMAs over K = 128 (eight K-steps of 16) into one accumulator, in one
// asm block: between MMAs only the 32-bit start-address words of the
// descriptors advance (shared-memory operands: address / 16, so a 32-byte
// step within a 128-byte swizzled row is +2 and a 4 KB step +256), which keeps
// the issuing thread's instruction count per MMA at three.  A from shared
// memory, K-major over two 16 KB halves (steps +2, +2, +2, +1018 to the next
// half, ...); B from shared memory with +256 per step.
__device__ __forceinline__ void mma8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, t;\n\t.reg .b32 al, ah, bl, bh;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p, %3, 0;\n\tsetp.eq.b32 t, 0, 0;\n\t"
      "mov.b64 {al, ah}, %1;\n\tmov.b64 {bl, bh}, %2;\n\t"
      "mov.b64 a, {al, ah};\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, p;\n\t"
      "add.u32 al, al, 2;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 a, {al, ah};\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, t;\n\t"
      "add.u32 al, al, 2;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 a, {al, ah};\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, t;\n\t"
      "add.u32 al, al, 2;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 a, {al, ah};\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, t;\n\t"
      "add.u32 al, al, 1018;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 a, {al, ah};\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, t;\n\t"
      "add.u32 al, al, 2;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 a, {al, ah};\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, t;\n\t"
      "add.u32 al, al, 2;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 a, {al, ah};\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, t;\n\t"
      "add.u32 al, al, 2;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 a, {al, ah};\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %4, t;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(accumulate), "r"(kIdesc)
      : "memory");
}

// The same with A in TMEM (eight columns per K-step: +8 to the TMEM address).
__device__ __forceinline__ void mma8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, t;\n\t.reg .b32 a, bl, bh;\n\t.reg .b64 b;\n\t"
      "setp.ne.b32 p, %3, 0;\n\tsetp.eq.b32 t, 0, 0;\n\t"
      "mov.b32 a, %1;\n\tmov.b64 {bl, bh}, %2;\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, p;\n\t"
      "add.u32 a, a, 8;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, t;\n\t"
      "add.u32 a, a, 8;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, t;\n\t"
      "add.u32 a, a, 8;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, t;\n\t"
      "add.u32 a, a, 8;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, t;\n\t"
      "add.u32 a, a, 8;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, t;\n\t"
      "add.u32 a, a, 8;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, t;\n\t"
      "add.u32 a, a, 8;\n\tadd.u32 bl, bl, 256;\n\tmov.b64 b, {bl, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %4, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(accumulate), "r"(kIdesc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// byte offset of the 16-byte chunk holding tokens t..t+7 (t % 8 == 0) of
// channel c in a K tile: MN-major over tokens, 1024-byte atoms of 8 channel
// rows x 64 tokens; atom (c/8, t/64) at ((c/8)*2 + t/64) * 1024
__device__ __forceinline__ uint32_t kt_off(int c, int t) {
  return uint32_t(((c >> 3) * 2 + (t >> 6)) * 1024 + (c & 7) * 128 +
                  ((((t & 63) >> 3) ^ (c & 7)) << 4));
}

// chunk of channels c..c+7 (c % 8 == 0) of token t in a V tile: MN-major over
// channels, atom (t/8, c/64) at ((t/8)*2 + c/64) * 1024
__device__ __forceinline__ uint32_t vt_off(int t, int c) {
  return uint32_t(((t >> 3) * 2 + (c >> 6)) * 1024 + (t & 7) * 128 +
                  ((((c & 63) >> 3) ^ (t & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  return h2u(__floats2half2_rn(a, b));
}

// ------------------------------------------------------------------ producers

// K tile: thread (c, qh) fills tokens [32q, 32q+32) of channel c for
// q = 2qh, 2qh+1.  Codes and (scale, zero) of the quantized part come from the ring
// stage `rs` (groups of the tile in order, [group][channel][kw words]); the
// bf16 tail, the active block and bits = 16 come straight from global memory.
// Byte offsets of the 16-byte chunks a K producer thread (c, qh) stores:
// chunk i (0..7) holds tokens 64 qh + 8 i .. +7 of channel c.
// Tiles whose K is wholly quantized are stored in the order the prmt-free
// dequantization produces: the token at tile position kpos(t) is t, permuted
// within groups of 16 (2-bit codes) or 8 (4-bit codes); 3-bit codes (32 to
// three words, two of them straddling words) are extracted one by one and
// keep the natural order.  V tiles hold their
// channels in the same kind of order for V's bit width (kpos<VB>, in every
// tile, bf16 rows included), so O's column kpos<VB>(c) is channel c and the
// epilogue reads it from there.  The V tile of such a
// tile puts token t's row at the same position, so P V pairs every score with
// its own value row; the softmax does not depend on column order.  Other
// tiles (K tail, active block, bf16 K) keep the natural order.
template <int KB>
__device__ __forceinline__ int kpos(int t) {
  if constexpr (KB == 2) return (t & ~15) | (8 * ((t >> 2) & 1) + 2 * (t & 3) + ((t >> 3) & 1));
  else if constexpr (KB == 4) return (t & ~7) | (2 * (t & 3) + ((t >> 2) & 1));
  else return t;
}

struct KOffsets {
  uint32_t o[8];
  uint32_t w[2], z[2];  // ring offsets of chunk 2qh+qi: code words (uint32), (scale, zero) pairs
  __device__ KOffsets(int c, int qh, int GK, int kw, int kb) {
    const uint32_t base = uint32_t(((c >> 3) * 2 + qh) * 1024 + (c & 7) * 128);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = base + uint32_t(((i ^ (c & 7)) & 7) << 4);
#pragma unroll
    for (int qi = 0; qi < 2; ++qi) {
      const int q = 2 * qh + qi;
      const int gi = (32 * q) / GK, off = (32 * q) % GK;
      w[qi] = uint32_t((gi * kHeadDim + c) * kw + off * kb / 32);
      z[qi] = uint32_t(gi * kHeadDim + c);
    }
  }
};

template <int KB, int VB>
__device__ __noinline__ void fill_k_general(const AttnArgs& a, const UnitLen ul, int u, int64_t tile_start,
                                            uint8_t* kt, const uint8_t* rs, int c, int qh);

// K tile, channel c, token chunks 2qh, 2qh+1.  The whole-quantized-tile case
// is inline; tiles that reach the bf16 tail or the active block take the
// out-of-line general path (at most two per call), which keeps the hot loop's
// code small.
template <int KB, int VB>
__device__ __forceinline__ void fill_k_tile(const AttnArgs& a, const UnitLen ul, int u, int64_t tile_start,
                                            uint8_t* kt, const uint8_t* rs, int c, int qh,
                                            const KOffsets& ko) {
  using ST = Stage<KB, VB>;
  const CacheView& cv = a.c;
  const int d = kHeadDim;
  if constexpr (KB < 16) {
    if (tile_start + TT <= ul.Lq) {
      // whole tile quantized: one 32-token chunk per iteration (a rolled
      // loop keeps the hot code small)
#pragma unroll 1
      for (int qi = 0; qi < 2; ++qi) {
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(rs + ST::kRKc) + (qi ? ko.w[1] : ko.w[0]);
        const __half2 sz = reinterpret_cast<const __half2*>(rs + ST::kRKsz)[qi ? ko.z[1] : ko.z[0]];
        const __half2 s2 = __half2half2(__low2half(sz));
        const __half2 z2 = __half2half2(__high2half(sz));
        uint4 out[4];  // tokens in kpos order
        if constexpr (KB == 4) {
          const uint4 w = *reinterpret_cast<const uint4*>(wp);
          out[0] = dequant4x8_raw(w.x, s2, z2);
          out[1] = dequant4x8_raw(w.y, s2, z2);
          out[2] = dequant4x8_raw(w.z, s2, z2);
          out[3] = dequant4x8_raw(w.w, s2, z2);
        } else if constexpr (KB == 3) {
          dequant3x32(wp[0], wp[1], wp[2], s2, z2, out);  // 4-byte aligned words
        } else {
          const uint2 w = *reinterpret_cast<const uint2*>(wp);
          dequant2x16_raw(w.x, s2, z2, out[0], out[1]);
          dequant2x16_raw(w.y, s2, z2, out[2], out[3]);
        }
        // chunk 1's offsets are chunk 0's shifted by +-64 bytes (bit 2 of the swizzle)
        uint8_t* dst = kt + (qi ? int(ko.o[4]) - int(ko.o[0]) : 0);
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(dst + ko.o[i]) = out[i];
      }
      // protected rows of this thread's two chunks
      const int* hdr = reinterpret_cast<const int*>(rs + ST::kRHdr);
      const int n = hdr[0], g0 = hdr[1], pbase = hdr[2];
      const int* rpos = reinterpret_cast<const int*>(rs + ST::kRPos);
      const uint16_t* rpk = reinterpret_cast<const uint16_t*>(rs + ST::kRPk);
      auto put = [&](int pos, uint16_t kv) {
        const int t = int(pos - tile_start);
        if (!DKV_IN_BOUNDS(t >= 0 && t < TT, cv.status)) return;
        if ((t >> 6) != qh) return;
        const int p = kpos<KB>(t);
        __half* dst = reinterpret_cast<__half*>(kt + kt_off(c, p & ~7)) + (p & 7);
        *dst = bf16_to_half(kv);
      };
      const int ns = n < ST::kProt ? n : ST::kProt;
#pragma unroll 1
      for (int i = 0; i < ns; ++i) {  // staged entries
        if (!DKV_IN_BOUNDS(g0 + i - pbase >= 0 && g0 + i - pbase < 32, cv.status)) break;
        put(rpos[g0 + i - pbase], rpk[i * d + c]);
      }
#pragma unroll 1
      for (int i = ns; i < n; ++i) {  // the rest from global memory
        if (!DKV_IN_BOUNDS(g0 + i < cv.P, cv.status)) break;
        put(__ldg(cv.prot_pos + size_t(u) * cv.P + g0 + i),
            __ldg(cv.prot_k + (size_t(u) * cv.P + g0 + i) * d + c));
      }
      return;
    }
  }
  fill_k_general<KB, VB>(a, ul, u, tile_start, kt, rs, c, qh);
}

template <int KB, int VB>
__device__ __noinline__ void fill_k_general(const AttnArgs& a, const UnitLen ul, int u, int64_t tile_start,
                                            uint8_t* kt, const uint8_t* rs, int c, int qh) {
  using ST = Stage<KB, VB>;
  const CacheView& cv = a.c;
  const int d = kHeadDim;
#pragma unroll 1
  for (int q = 2 * qh; q < 2 * qh + 2; ++q) {
    const int64_t pos0 = tile_start + 32 * q;
    uint4 out[4];
    const uint16_t* raw = nullptr;
    bool codes = false;
    if (pos0 < ul.Lq) {
      if constexpr (KB < 16) codes = true;
      else raw = cv.k_raw + (size_t(u) * cv.cap + pos0) * d;
    } else if (pos0 < ul.L) {
      raw = cv.k_tail + (size_t(u) * cv.GK + (pos0 - ul.Lq)) * d;
    } else if (pos0 < ul.n_tok) {
      raw = a.k_act + (size_t(u) * cv.blk + (pos0 - ul.L)) * d;
    }
    if (codes) {
      if constexpr (KB < 16) {
        const int gi = (32 * q) / cv.GK;  // group within the tile
        const int o = (32 * q) % cv.GK;
        const uint32_t* kc = reinterpret_cast<const uint32_t*>(rs + ST::kRKc) +
                             (gi * d + c) * cv.kw + o * KB / 32;
        const __half2 sz = reinterpret_cast<const __half2*>(rs + ST::kRKsz)[gi * d + c];
        const __half2 s2 = __half2half2(__low2half(sz));
        const __half2 z2 = __half2half2(__high2half(sz));
        if constexpr (KB == 4) {
          const uint4 w = *reinterpret_cast<const uint4*>(kc);
          out[0] = dequant4x8(w.x, s2, z2);
          out[1] = dequant4x8(w.y, s2, z2);
          out[2] = dequant4x8(w.z, s2, z2);
          out[3] = dequant4x8(w.w, s2, z2);
        } else if constexpr (KB == 3) {
          dequant3x32(kc[0], kc[1], kc[2], s2, z2, out);
        } else {
          const uint2 w = *reinterpret_cast<const uint2*>(kc);
          dequant2x16(w.x, s2, z2, out[0], out[1]);
          dequant2x16(w.y, s2, z2, out[2], out[3]);
        }
      }
    } else if (raw) {
      uint32_t h[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float lo = __uint_as_float(uint32_t(__ldg(raw + size_t(2 * t) * d + c)) << 16);
        const float hi = __uint_as_float(uint32_t(__ldg(raw + size_t(2 * t + 1) * d + c)) << 16);
        h[t] = pack_h2(lo, hi);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(kt + kt_off(c, 32 * q + 8 * i)) = out[i];
    if constexpr (KB < 16) {
      if (codes) {
        // protected rows of this chunk: their bf16 K from the staged side-table
        // slice (entries past the staged ones from global memory)
        const int* hdr = reinterpret_cast<const int*>(rs + ST::kRHdr);
        const int n = hdr[0], g0 = hdr[1], pbase = hdr[2];
        const int* rpos = reinterpret_cast<const int*>(rs + ST::kRPos);
        const uint16_t* rpk = reinterpret_cast<const uint16_t*>(rs + ST::kRPk);
        for (int i = 0; i < n; ++i) {
          if (!DKV_IN_BOUNDS(i < ST::kProt ? g0 + i - pbase >= 0 && g0 + i - pbase < 32
                                             : g0 + i < cv.P, cv.status))
            break;
          const int pos = i < ST::kProt ? rpos[g0 + i - pbase]
                                          : __ldg(cv.prot_pos + size_t(u) * cv.P + g0 + i);
          if (pos >= pos0 && pos < pos0 + 32) {
            const int t = 32 * q + int(pos - pos0);
            const uint16_t kv = i < ST::kProt
                                    ? rpk[i * d + c]
                                    : __ldg(cv.prot_k + (size_t(u) * cv.P + g0 + i) * d + c);
            __half* dst = reinterpret_cast<__half*>(kt + kt_off(c, t & ~7)) + (t & 7);
            *dst = bf16_to_half(kv);
          }
        }
      }
    }
  }
}

// V tile: thread `tid` (0..255) fills items (token t, channel quarter qq) with
// qq = tid % 4 and t = v_slot_token(tid / 4) + 64 r (r = 0, 1): a warp reads
// its eight tokens' code words from the ring stage ([token][vw words]) in
// 32-byte pieces or larger.

// Token (0..63 of a half tile) whose V row the V producer slot s (= tid / 4,
// four threads per token) fills.  In the K tile's row order (kpos) tokens t
// and t + 1 sit 2 rows apart modulo 8, which gives their 16-byte chunks the
// same bank groups; a quarter warp (two slots) therefore takes tokens t and
// t + 8 (2-bit K) or t + 4 (4-bit K), which sit 1 row apart modulo 8, and
// its eight 16-byte stores fall in eight distinct bank groups.
template <int KB>
__device__ __forceinline__ int v_slot_token(int s) {
  if constexpr (KB == 2) return (s & ~15) | ((s & 15) >> 1) | ((s & 1) << 3);
  else if constexpr (KB == 4) return (s & ~7) | ((s & 7) >> 1) | ((s & 1) << 2);
  else return s;
}

// Byte offsets of the 16-byte chunks a V producer thread stores: item r
// (token t0 + 64 r, quarter tid & 3), store i = chunk (i + rot) & 3.
template <int KB>
struct VOffsets {
  uint32_t base, x[4];
  uint32_t w[2], z[2];  // ring offsets of item r: code words (uint32), (scale, zero) pairs
  __device__ VOffsets(int tid, int vw, int vgroups, int GV, int vb) {
    // row of this thread's token t0 (and t0 + 64): its kpos position
    // (identity for bf16 K)
    const int t0 = v_slot_token<KB>(tid >> 2);
    const int p = kpos<KB>(t0);
    const int qq = tid & 3, t7 = p & 7, rot = qq & 2;
    base = uint32_t(((p >> 3) * 2 + (qq >> 1)) * 1024 + t7 * 128);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = uint32_t(((4 * (qq & 1) + ((i + rot) & 3)) ^ t7) << 4);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int t = t0 + 64 * r;
      w[r] = uint32_t(t * vw + qq * (vb < 16 ? vb : 0));  // a channel quarter: vb words
      z[r] = uint32_t(t * vgroups + (qq * 32) / GV);
    }
  }
};

template <int KB, int VB>
__device__ __noinline__ void fill_v_general(const AttnArgs& a, const UnitLen ul, int u, int64_t tile_start,
                                            uint8_t* vt, const uint8_t* rs, int tid, int perm_kb);

// V tile: the whole-quantized-tile case inline, the rest out of line.  Rows
// follow the K tile's order: kpos when the tile's K is wholly quantized.
template <int KB, int VB, bool SINK>
__device__ __forceinline__ void fill_v_tile(const AttnArgs& a, const UnitLen ul, int u, int64_t tile_start,
                                            uint8_t* vt, const uint8_t* rs, int tid,
                                            const VOffsets<KB>& vo) {
  using ST = Stage<KB, VB>;
  const CacheView& cv = a.c;
  const bool k_whole = KB < 16 && tile_start + TT <= ul.Lq;
  if constexpr (VB < 16) {
    // (with a sink, tiles holding sink positions take the general path, which
    // reads their bf16 rows)
    if ((KB < 16 ? k_whole : tile_start + TT <= ul.L) && (!SINK || tile_start >= cv.sink)) {
      // whole tile quantized: one item per iteration (a rolled loop keeps
      // the hot code small)
      const bool rot = (tid & 2) != 0;
#pragma unroll 1
      for (int r = 0; r < 2; ++r) {
        const uint32_t* xp = reinterpret_cast<const uint32_t*>(rs + ST::kRVc) + (r ? vo.w[1] : vo.w[0]);
        const __half2 sz = reinterpret_cast<const __half2*>(rs + ST::kRVsz)[r ? vo.z[1] : vo.z[0]];
        const __half2 s2 = __half2half2(__low2half(sz));
        const __half2 z2 = __half2half2(__high2half(sz));
        uint4 out[4];  // channels in kpos<VB> order
        if constexpr (VB == 3) {
          uint4 nat[4];  // 4-byte aligned words; channels in natural order
          dequant3x32(xp[0], xp[1], xp[2], s2, z2, nat);
          out[0] = rot ? nat[2] : nat[0];
          out[1] = rot ? nat[3] : nat[1];
          out[2] = rot ? nat[0] : nat[2];
          out[3] = rot ? nat[1] : nat[3];
        } else if constexpr (VB == 4) {
          uint4 x = *reinterpret_cast<const uint4*>(xp);
          if (rot) x = make_uint4(x.z, x.w, x.x, x.y);
          out[0] = dequant4x8_raw(x.x, s2, z2);
          out[1] = dequant4x8_raw(x.y, s2, z2);
          out[2] = dequant4x8_raw(x.z, s2, z2);
          out[3] = dequant4x8_raw(x.w, s2, z2);
        } else {
          uint2 x = *reinterpret_cast<const uint2*>(xp);
          if (rot) x = make_uint2(x.y, x.x);
          dequant2x16_raw(x.x, s2, z2, out[0], out[1]);
          dequant2x16_raw(x.y, s2, z2, out[2], out[3]);
        }
        uint8_t* dst = vt + vo.base + 16384u * uint32_t(r);
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(dst + vo.x[i]) = out[i];
      }
      return;
    }
  }
  fill_v_general<KB, VB>(a, ul, u, tile_start, vt, rs, tid, k_whole ? KB : 16);
}

template <int KB, int VB>
__device__ __noinline__ void fill_v_general(const AttnArgs& a, const UnitLen ul, int u, int64_t tile_start,
                                            uint8_t* vt, const uint8_t* rs, int tid, int perm_kb) {
  using ST = Stage<KB, VB>;  // KB: the ring stage's layout (the row order is perm_kb)
  const CacheView& cv = a.c;
  const int d = kHeadDim;
#pragma unroll 1
  for (int r = 0; r < 2; ++r) {
    const int sl = tid >> 2, qq = tid & 3;
    const int t = (perm_kb == 2 ? v_slot_token<2>(sl) : (perm_kb == 4 ? v_slot_token<4>(sl) : sl)) +
                  64 * r;
    const int64_t pos = tile_start + t;
    // row of token t (the K tile's order, see kpos)
    const int p = perm_kb == 2 ? kpos<2>(t) : (perm_kb == 4 ? kpos<4>(t) : t);
    uint4 out[4];
    const uint16_t* raw = nullptr;
    bool codes = false;
    if (pos < ul.L) {
      if constexpr (VB < 16) {
        if (pos < cv.sink) raw = cv.v_sink + (size_t(u) * cv.sink + size_t(pos)) * d;  // sink row
        else codes = true;
      } else {
        raw = cv.v_raw + (size_t(u) * cv.cap + pos) * d;
      }
    } else if (pos < ul.n_tok) {
      raw = a.v_act + (size_t(u) * cv.blk + (pos - ul.L)) * d;
    }
    // out[i] holds channels 32qq + 8((i + rot) & 3): lanes of a quarter warp
    // (two tokens one row apart modulo 8, see v_slot_token, x quarters 0..3)
    // then store to 8 distinct bank groups
    const int rot = qq & 2;
    if (codes) {
      if constexpr (VB < 16) {
        const __half2 sz =
            reinterpret_cast<const __half2*>(rs + ST::kRVsz)[t * cv.vgroups + (qq * 32) / cv.GV];
        const __half2 s2 = __half2half2(__low2half(sz));
        const __half2 z2 = __half2half2(__high2half(sz));
        const uint32_t* vc = reinterpret_cast<const uint32_t*>(rs + ST::kRVc) + t * cv.vw;
        if constexpr (VB == 3) {
          uint4 nat[4];
          dequant3x32(vc[qq * 3], vc[qq * 3 + 1], vc[qq * 3 + 2], s2, z2, nat);
          out[0] = rot ? nat[2] : nat[0];
          out[1] = rot ? nat[3] : nat[1];
          out[2] = rot ? nat[0] : nat[2];
          out[3] = rot ? nat[1] : nat[3];
        } else if constexpr (VB == 4) {
          uint4 w = *reinterpret_cast<const uint4*>(vc + qq * 4);
          if (rot) w = make_uint4(w.z, w.w, w.x, w.y);
          out[0] = dequant4x8_raw(w.x, s2, z2);
          out[1] = dequant4x8_raw(w.y, s2, z2);
          out[2] = dequant4x8_raw(w.z, s2, z2);
          out[3] = dequant4x8_raw(w.w, s2, z2);
        } else {
          uint2 w = *reinterpret_cast<const uint2*>(vc + qq * 2);
          if (rot) w = make_uint2(w.y, w.x);
          dequant2x16_raw(w.x, s2, z2, out[0], out[1]);
          dequant2x16_raw(w.y, s2, z2, out[2], out[3]);
        }
      }
    } else if (raw) {
      uint4 nat[4];  // channels 32qq + 8k .. + 7, natural order
#pragma unroll
      for (int k = 0; k < 4; ++k)
        nat[k] = bf16x8_to_f16x8(__ldg(reinterpret_cast<const uint4*>(raw + qq * 32 + 8 * k)));
      uint4 pc[4];  // the same channels in kpos<VB> order (the quantized rows' order)
      if constexpr (VB == 4) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          pc[k] = make_uint4(prmt(nat[k].x, nat[k].z, 0x5410), prmt(nat[k].x, nat[k].z, 0x7632),
                             prmt(nat[k].y, nat[k].w, 0x5410), prmt(nat[k].y, nat[k].w, 0x7632));
      } else if constexpr (VB == 2) {
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint4 A = nat[2 * g], B = nat[2 * g + 1];
          pc[2 * g] = make_uint4(prmt(A.x, B.x, 0x5410), prmt(A.x, B.x, 0x7632),
                                 prmt(A.y, B.y, 0x5410), prmt(A.y, B.y, 0x7632));
          pc[2 * g + 1] = make_uint4(prmt(A.z, B.z, 0x5410), prmt(A.z, B.z, 0x7632),
                                     prmt(A.w, B.w, 0x5410), prmt(A.w, B.w, 0x7632));
        }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) pc[k] = nat[k];
      }
      // rot is 0 or 2
      out[0] = rot ? pc[2] : pc[0];
      out[1] = rot ? pc[3] : pc[1];
      out[2] = rot ? pc[0] : pc[2];
      out[3] = rot ? pc[1] : pc[3];
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(vt + vt_off(p, 32 * qq + 8 * ((i + rot) & 3))) = out[i];
  }
}

// ------------------------------------------------------------ shared pipeline loops

// Shared-memory addresses of one kernel's pipeline: the ring of packed
// tiles, the two dequantized K and V tile buffers, and the barriers that
// hand them over (entry i of a barrier pair or ring at +8 i).
struct Pipe {
  uint8_t* sm;
  uint32_t sm_base;
  uint32_t ring;              // offset of ring stage 0 (stages Stage<KB, VB>::kBytes apart)
  uint32_t k_buf0, v_buf0;    // offsets of K / V tile buffer 0 (buffer 1 at + kTileBytes)
  uint32_t kfull, kempty, vfull, vempty, rfull, rempty;  // barrier addresses
};

// K producer thread pt (0..255): channel pt % 128, token chunks 2 qh, 2 qh + 1
// of every tile, qh = pt / 128.
template <int KB, int VB, int STAGES>
__device__ __forceinline__ void k_producer_loop(const AttnArgs& a, const UnitLen* uls, int u,
                                                int64_t t_begin, int nt, const Pipe& p,
                                                volatile int* abort_flag, int pt) {
  using ST = Stage<KB, VB>;
  const CacheView& cv = a.c;
  const int c = pt & 127;   // channel
  const int qh = pt >> 7;   // chunks 2qh, 2qh+1 of each tile
  const KOffsets ko(c, qh, cv.GK, cv.kw, KB < 16 ? KB : 16);
#pragma unroll 1
  for (int j = 0; j < nt; ++j) {
    const int b = j & 1, st = j % STAGES;
    if (!mbar_wait_fast(p.kempty + 8u * b, ((j >> 1) & 1) ^ 1, a, abort_flag)) break;
    if (!mbar_wait_fast(p.rfull + 8u * st, (j / STAGES) & 1, a, abort_flag)) break;
    if (pt == 0) DKV_TR(1, j);
    fill_k_tile<KB, VB>(a, *uls, u, (t_begin + j) * TT, p.sm + p.k_buf0 + b * kTileBytes,
                    p.sm + p.ring + st * ST::kBytes, c, qh, ko);
    fence_async_smem();
    if (pt == 0) DKV_TR(2, j);
    mbar_arrive(p.kfull + 8u * b);
    mbar_arrive(p.rempty + 8u * st);
  }
}

// V producer thread pt (0..255).
template <int KB, int VB, bool SINK, int STAGES>
__device__ __forceinline__ void v_producer_loop(const AttnArgs& a, const UnitLen* uls, int u,
                                                int64_t t_begin, int nt, const Pipe& p,
                                                volatile int* abort_flag, int pt) {
  using ST = Stage<KB, VB>;
  const CacheView& cv = a.c;
  const VOffsets<KB> vo(pt, cv.vw, cv.vgroups, cv.GV, VB < 16 ? VB : 16);
#pragma unroll 1
  for (int j = 0; j < nt; ++j) {
    const int b = j & 1, st = j % STAGES;
    if (!mbar_wait_fast(p.vempty + 8u * b, ((j >> 1) & 1) ^ 1, a, abort_flag)) break;
    if (pt == 0) DKV_TR(11, j);
    if (!mbar_wait_fast(p.rfull + 8u * st, (j / STAGES) & 1, a, abort_flag)) break;
    if (pt == 0) DKV_TR(3, j);
    fill_v_tile<KB, VB, SINK>(a, *uls, u, (t_begin + j) * TT, p.sm + p.v_buf0 + b * kTileBytes,
                              p.sm + p.ring + st * ST::kBytes, pt, vo);
    fence_async_smem();
    if (pt == 0) DKV_TR(4, j);
    mbar_arrive(p.vfull + 8u * b);
    mbar_arrive(p.rempty + 8u * st);
  }
}

// Loader warp: lanes prefetch the side-table group index of 32 tiles at a
// time; lane 0 issues the bulk copies of each tile into the ring.  Token
// positions fit in 32 bits (capacity <= 2^30) and K groups are 32, 64 or 128
// tokens, so the group arithmetic is 32-bit shifts.
template <int KB, int VB, int STAGES>
__device__ __forceinline__ void loader_loop(const AttnArgs& a, const UnitLen* uls, int u,
                                            int64_t t_begin, int nt, const Pipe& p,
                                            volatile int* abort_flag, int lane) {
  using ST = Stage<KB, VB>;
  const CacheView& cv = a.c;
  const int gks = KB < 16 ? __ffs(cv.GK) - 1 : 0;
  const int Lq = uls->Lq, Lc = uls->L, t0 = int(t_begin) * TT;
  const int32_t* gs = cv.prot_gstart + size_t(u) * size_t(cv.nG + 1);
  int issued = 0;     // tiles 0 .. issued-1 went through the ring
  int stalled = -1;   // (bounds-checking build) the tile whose copies were withheld
  int pf0 = 0, pf1 = 0;  // this lane's prefetched gstart values (tile j0 + lane)
#pragma unroll 1
  for (int j = 0; j < nt; ++j) {
    if constexpr (KB < 16) {
      if ((j & 31) == 0) {
        pf0 = pf1 = 0;
        const int jj = j + lane;
        const int ts = t0 + jj * TT;
        if (jj < nt && ts < Lq && cv.P > 0) {
          const int q_end = ts + TT < Lq ? ts + TT : Lq;
          pf0 = __ldg(gs + (ts >> gks));
          pf1 = __ldg(gs + (q_end >> gks));
        }
      }
    }
    const int g0 = __shfl_sync(0xffffffffu, pf0, j & 31);
    const int g1 = __shfl_sync(0xffffffffu, pf1, j & 31);
    const int st = j % STAGES;
    const uint32_t rfull = p.rfull + 8u * st;
    if (!__all_sync(0xffffffffu, mbar_wait_fast(p.rempty + 8u * st, ((j / STAGES) & 1) ^ 1, a, abort_flag)))
      break;
    if (lane == 0) DKV_TR(0, j);
    ++issued;
#ifdef DKV_BOUNDS_CHECK
    if (j == a.test_stall_tile) {
      // test hook: nothing is copied and nothing arrives on this stage, so
      // the producers' bounded waits on it run out (DKV_FLAG_TIMEOUT)
      stalled = j;
      continue;
    }
#endif
    if (lane == 0) {
      const int ts = t0 + j * TT;
      const uint32_t dst = p.sm_base + p.ring + st * ST::kBytes;
      uint32_t kc_b = 0, ksz_b = 0, vc_b = 0, vsz_b = 0, pos_b = 0, pk_b = 0;
      int g_lo = 0, pidx0 = 0;  // pidx0: first staged position, relative to the unit
      const int n = g1 - g0;
      if (KB < 16 && ts < Lq) {
        g_lo = ts >> gks;
        const int q_end = ts + TT < Lq ? ts + TT : Lq;  // multiple of GK
        const uint32_t ng = uint32_t((q_end >> gks) - g_lo);
        kc_b = ng * kHeadDim * uint32_t(cv.kw) * 4u;
        ksz_b = ng * kHeadDim * 4u;
        if (n > 0) {
          const int nst = n < ST::kProt ? n : ST::kProt;
          // 16-byte aligned superset of the staged positions (the unit's
          // slice starts at u * P entries)
          const int64_t e0 = int64_t(u) * cv.P + g0;
          const int64_t ea = e0 & ~int64_t(3);
          pidx0 = int(ea - int64_t(u) * cv.P);
          pos_b = uint32_t(((e0 + nst + 3) & ~int64_t(3)) - ea) * 4u;
          pk_b = uint32_t(nst) * kHeadDim * 2u;
        }
      }
      if (VB < 16 && ts < Lc) {
        const uint32_t nv = uint32_t((ts + TT < Lc ? ts + TT : Lc) - ts);
        vc_b = nv * uint32_t(cv.vw) * 4u;
        vsz_b = nv * uint32_t(cv.vgroups) * 4u;
      }
      const size_t ug = size_t(u) * size_t(cv.nG) + size_t(g_lo);
      {
        // bounds-checking build: each copy inside its buffer and its ring
        // slot, else left out (the staged side table with it); the byte
        // counts stay consistent with the expect_tx below
        const size_t U = size_t(cv.U), P = size_t(cv.P), e = size_t(u) * P;
        if (kc_b && !DKV_IN_BOUNDS(
                        kc_b <= ST::kRKsz - ST::kRKc && ksz_b <= ST::kRHdr - ST::kRKsz &&
                        (ug * kHeadDim * cv.kw) * 4 + kc_b <= U * cv.nG * kHeadDim * cv.kw * 4 &&
                        (ug * kHeadDim) * 4 + ksz_b <= U * cv.nG * kHeadDim * 4, cv.status))
          kc_b = ksz_b = pos_b = pk_b = 0;
        // (the staged positions are a 16-byte aligned superset: up to three
        // entries before and after the unit's slice, inside the arena)
        if (pos_b && !DKV_IN_BOUNDS(
                         g0 >= 0 && int64_t(e) + pidx0 >= 0 &&
                         pos_b <= ST::kRPk - ST::kRPos &&
                         pk_b <= ST::kRVc - ST::kRPk &&
                         (e + size_t(pidx0)) * 4 + pos_b <= (U * P + 3) * 4 &&
                         (e + size_t(g0)) * kHeadDim * 2 + pk_b <= U * P * kHeadDim * 2, cv.status))
          pos_b = pk_b = 0;
        const size_t ut = size_t(u) * size_t(cv.cap) + size_t(ts);
        if (vc_b && !DKV_IN_BOUNDS(
                        vc_b <= ST::kRVsz - ST::kRVc && vsz_b <= ST::kBytes - ST::kRVsz &&
                        ut * cv.vw * 4 + vc_b <= U * size_t(cv.cap) * cv.vw * 4 &&
                        ut * cv.vgroups * 4 + vsz_b <= U * size_t(cv.cap) * cv.vgroups * 4, cv.status))
          vc_b = vsz_b = 0;
      }
      int* hdr = reinterpret_cast<int*>(p.sm + p.ring + st * ST::kBytes + ST::kRHdr);
      hdr[0] = pos_b ? n : 0;  // pos_b is set exactly when the tile has protected rows
      hdr[1] = g0;
      hdr[2] = pidx0;
      mbar_arrive_expect_tx(rfull, kc_b + ksz_b + vc_b + vsz_b + pos_b + pk_b);
      if (kc_b) {
        bulk_g2s(dst + ST::kRKc, cv.k_codes + ug * kHeadDim * cv.kw, kc_b, rfull);
        bulk_g2s(dst + ST::kRKsz, cv.k_sz + ug * kHeadDim, ksz_b, rfull);
      }
      if (pos_b) {
        const size_t e = size_t(u) * size_t(cv.P);
        bulk_g2s(dst + ST::kRPos, cv.prot_pos + e + size_t(pidx0), pos_b, rfull);
        bulk_g2s(dst + ST::kRPk, cv.prot_k + (e + size_t(g0)) * kHeadDim, pk_b, rfull);
      }
      if (vc_b) {
        const size_t ut = size_t(u) * size_t(cv.cap) + size_t(ts);
        bulk_g2s(dst + ST::kRVc, cv.v_codes + ut * cv.vw, vc_b, rfull);
        bulk_g2s(dst + ST::kRVsz, cv.v_sz + ut * cv.vgroups, vsz_b, rfull);
      }
    }
    __syncwarp();
  }
  // drain: the last copies issued have landed before shared memory is released
  if (lane == 0)
    for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j)
      if (j != stalled) mbar_wait(p.rfull + 8u * (j % STAGES), (j / STAGES) & 1, a, abort_flag, true);
}

// ------------------------------------------------------------------ kernel

template <int KB, int VB, bool SINK>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sm_base = smem_u32(sm);
  const uint32_t bar0 = sm_base + SmemTail<KB, VB>::kBar;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SmemTail<KB, VB>::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SmemTail<KB, VB>::kMisc + 4);

  const CacheView& cv = a.c;
  // CTA = (unit, split, row block): a query group of more than 128 rows is
  // cut into row blocks of rows/nrb; smaller blocks are zero-padded to M = 128
  const int nrb = (cv.rows + 127) / 128;
  const int rpb = cv.rows / nrb;
  const int rb = blockIdx.x % nrb;
  const int u = (blockIdx.x / nrb) / a.nsplit;
  const int sp = (blockIdx.x / nrb) % a.nsplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const UnitLen ul = unit_len(a, u);  // this unit's sequence length
  const int64_t n_tiles = (ul.n_tok + TT - 1) / TT;
  const int64_t t_begin = int64_t(sp) * a.tiles_per_split;
  const int64_t t_end = t_begin + a.tiles_per_split < n_tiles ? t_begin + a.tiles_per_split : n_tiles;
  const int nt = t_end > t_begin ? int(t_end - t_begin) : 0;
  if (nt == 0) {
    // a split past the end of a shorter sequence (the plan follows the
    // longest): an empty partial -- max -inf, sum 0, O = 0 -- which the
    // combine gives weight 0.  (With one split every unit has tiles.)
    pdl_wait();
    pdl_trigger();
    if (!a.final_out) {
      const size_t prow = (size_t(u) * a.part_stride + a.part_base + sp) * cv.rows + size_t(rb) * rpb;
      for (int i = threadIdx.x; i < rpb * (kHeadDim / 8); i += kThreads)
        reinterpret_cast<uint4*>(a.part_o + prow * kHeadDim)[i] = make_uint4(0u, 0u, 0u, 0u);
      for (int i = threadIdx.x; i < rpb; i += kThreads)
        a.part_ml[prow + i] = make_float2(-__int_as_float(0x7f800000), 0.f);
    }
    return;
  }

  // the unit's lengths live in shared memory from here on: read where used,
  // not held in registers through the role loops
  const UnitLen* uls = reinterpret_cast<const UnitLen*>(sm + SmemTail<KB, VB>::kMisc + 16);
  const Pipe pipe{sm, sm_base, Smem::kRing, Smem::kK0, Smem::kV0, bar(KFULL), bar(SFULL),
                  bar(VFULL), bar(VEMPTY), bar(RFULL), bar(REMPTY)};
  if (threadIdx.x == 0) {
    *reinterpret_cast<UnitLen*>(sm + SmemTail<KB, VB>::kMisc + 16) = ul;
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(KFULL + b), 256);
      mbar_init(bar(VFULL + b), 256);
      mbar_init(bar(VEMPTY + b), 1);
      mbar_init(bar(SFULL + b), 1);  // also tells the K producers that K_b is free
      mbar_init(bar(SFREE + b), 128);
      mbar_init(bar(PFULL + b), 128);
      mbar_init(bar(RREADY + b), 128);
    }
    mbar_init(bar(QREADY), 256);
    mbar_init(bar(LSUM), 256);
    mbar_init(bar(DONE), 1);
    for (int st = 0; st < kStages; ++st) {
      mbar_init(bar(RFULL + st), 1);
      mbar_init(bar(REMPTY + st), 512);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  pdl_wait();  // no global memory access above this line
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) DKV_TR(9, 0);
  const uint32_t tmem = *tmem_slot;

  if (warp < 8) {
    // ------------------------------------------------------------ softmax
    regs_inc<kRegSoftmax>();
    const int lr = threadIdx.x & 127;   // TMEM lane = row of this block
    const int h = threadIdx.x >> 7;     // warpgroup: tiles j = h (mod 2); Q / output half h
    const bool row_ok = lr < rpb;       // padding rows carry Q = 0 and write nothing
    // a warp holding only padding rows skips the softmax arithmetic (its P
    // rows feed only padding rows of O, which are never read)
    const bool warp_rows = (warp & 3) * 32 < rpb;
    const int r = rb * rpb + lr;        // query row of the unit
    const uint32_t lane_base = tmem + (uint32_t((warp & 3) * 32) << 16);
    float* ref = reinterpret_cast<float*>(sm + SmemTail<KB, VB>::kRef);    // [tile parity][row]
    float* lsum = reinterpret_cast<float*>(sm + SmemTail<KB, VB>::kLsum);  // [warpgroup][row], then refs
    // a negative scale is folded into Q (an exact fp16 sign flip), so scores
    // are always multiplied by sc > 0; scale 0 (uniform weights) uses 1e-30
    const bool qneg = a.scale_log2 < 0.f;
    const float sc = fmaxf(fabsf(a.scale_log2), 1e-30f);
    {
      const uint4* qrow = reinterpret_cast<const uint4*>(
          a.q + (size_t(u) * cv.rows + (row_ok ? r : 0)) * kHeadDim + 64 * h);
      uint32_t qv[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 y = row_ok ? bf16x8_to_f16x8(__ldg(qrow + i)) : make_uint4(0u, 0u, 0u, 0u);
        if (qneg) y = make_uint4(y.x ^ 0x80008000u, y.y ^ 0x80008000u, y.z ^ 0x80008000u,
                                 y.w ^ 0x80008000u);
        qv[4 * i + 0] = y.x;
        qv[4 * i + 1] = y.y;
        qv[4 * i + 2] = y.z;
        qv[4 * i + 3] = y.w;
      }
      // row lr, channels [64h, 64h + 64): the 16-byte chunk c of the row at
      // chunk c ^ (row mod 8) of its 128-byte line (K-major, 128-byte swizzle)
      uint8_t* qh = sm + Smem::kQ + h * 16384 + lr * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(qh + ((c ^ (lr & 7)) << 4)) =
            make_uint4(qv[4 * c], qv[4 * c + 1], qv[4 * c + 2], qv[4 * c + 3]);
      fence_async_smem();
      mbar_arrive(bar(QREADY));
    }
    // Every tile j has one reference max per row, r_j (log2 units), non-
    // decreasing in j: r_j = r_(j-1) unless the tile's max exceeds it by more
    // than 8 (P <= 2^8), then r_j = max(r_(j-1), tile max).  O always holds
    // its sum relative to the reference of the last PV; this warpgroup's row
    // sum l is relative to r_w, the reference of its own last tile.
    float r_w = -__int_as_float(0x7f800000);
    float l = 0.f;
    bool ok = true;
#pragma unroll 1
    for (int j = h; j < nt && ok; j += 2) {
      const int b = h;  // S and P buffers, reference slot and barriers of this warpgroup's tiles
      const uint32_t s_col = b ? kColS1 : kColS0, p_col = b ? kColP1 : kColP0;
      // tcgen05.ld/st are warp-collective: every branch around them is warp-uniform
      if (!__all_sync(0xffffffffu, mbar_wait(bar(SFULL + b), (j >> 1) & 1, a, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if ((threadIdx.x & 127) == 0) DKV_TR(6, j);
      if (!warp_rows) {
        // Arrivals for tile j only once PV(j-2) is complete (so are all
        // arrivals for tile j-2): QK(j) can complete while the row warps are
        // still in tile j-2 after their SFREE, and early arrivals here would
        // count toward tile j-2's RREADY / PFULL phases.
        if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar(VEMPTY + b), ((j - 2) >> 1) & 1, a,
                                                          abort_flag))) {
          ok = false;
          break;
        }
        mbar_arrive(bar(RREADY + b));
        mbar_arrive(bar(SFREE + b));
        mbar_arrive(bar(PFULL + b));
        continue;
      }
      const int64_t tile_start = (t_begin + j) * TT;
      const int n_tok = uls->n_tok;
      const int valid = n_tok - tile_start < TT ? int(n_tok - tile_start) : TT;
      // Token counts are multiples of 32, so a tile holds n32 = valid / 32
      // whole 32-column chunks of scores; columns past them are never read
      // (and the PV MMAs stop at the same token).
      const int n32 = valid >> 5;
      // pass 1: max of the raw scores, two chunks per wait (an odd last chunk
      // is loaded twice, which leaves the max unchanged)
      float pm = -__int_as_float(0x7f800000);
#pragma unroll 1
      for (int cc = 0; cc < n32; cc += 2) {
        uint32_t sv[32], sw[32];
        tmem_ld32(lane_base + s_col + 32 * cc, sv);
        tmem_ld32(lane_base + s_col + 32 * (cc + 1 < n32 ? cc + 1 : cc), sw);
        tmem_ld_wait();
        float m4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) m4[i] = fmaxf(__uint_as_float(sv[i]), __uint_as_float(sw[i]));
#pragma unroll
        for (int i = 4; i < 32; ++i)
          m4[i & 3] = max3f(m4[i & 3], __uint_as_float(sv[i]), __uint_as_float(sw[i]));
        pm = max3f(pm, fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
      const float mx = pm * sc;
      // the previous tile's reference (bounded wait on the other warpgroup)
      float r_prev = -__int_as_float(0x7f800000);
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar(RREADY + (b ^ 1)), ((j - 1) >> 1) & 1,
                                               a, abort_flag))) {
          ok = false;
          break;
        }
        r_prev = ref[(b ^ 1) * 128 + lr];
      }
      // lazy rescale, decided per warp; rows whose max did not grow keep r_prev
      if ((threadIdx.x & 127) == 0) DKV_TR(12, j);
      const bool rescale = __any_sync(0xffffffffu, mx > r_prev + 8.f);
      const float r_j = rescale ? fmaxf(r_prev, mx) : r_prev;
      ref[b * 128 + lr] = r_j;
      mbar_arrive(bar(RREADY + b));
      l *= fast_exp2(r_w - r_j);  // 1 when unchanged, 0 on this warpgroup's first tile
      r_w = r_j;
      // pass 2: P = 2^(s*sc - r_j) as fp16 pairs into P_b, once PV(j-2) has
      // read it (QK(j) is issued before PV(j-2)); 16-column chunks, the load
      // of chunk c+1 in flight while chunk c is computed; S_b is released to
      // QK(j+2) after its last load
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar(VEMPTY + b), ((j - 2) >> 1) & 1, a,
                                                        abort_flag))) {
        ok = false;
        break;
      }
      const uint64_t sc2 = f2pack(sc, sc), nm2 = f2pack(-r_j, -r_j);
      uint64_t l2[2] = {0ull, 0ull};  // two packed pairs of partial row sums
      uint32_t va[16], vb[16];
      auto chunk = [&](const uint32_t (&v)[16], int c) {
        uint32_t pv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float x0, x1;
          f2unpack(ffma2(f2pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), sc2, nm2),
                   x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          l2[i & 1] = fadd2(l2[i & 1], f2pack(p0, p1));
          pv[i] = pack_h2(p0, p1);
        }
        tmem_st8(lane_base + p_col + 8 * c, pv);
      };
      const int n16 = 2 * n32;
      tmem_ld16(lane_base + s_col, va);
      tmem_ld_wait();
#pragma unroll 1
      for (int c = 0; c < n16; c += 2) {
        tmem_ld16(lane_base + s_col + 16 * (c + 1), vb);
        chunk(va, c);
        tmem_ld_wait();
        if (c + 2 < n16) {
          tmem_ld16(lane_base + s_col + 16 * (c + 2), va);
        } else {
          tc_fence_before();
          mbar_arrive(bar(SFREE + b));
        }
        chunk(vb, c + 1);
        if (c + 2 < n16) tmem_ld_wait();
      }
      {
        float a0, a1, b0, b1;
        f2unpack(l2[0], a0, a1);
        f2unpack(l2[1], b0, b1);
        l += (a0 + b0) + (a1 + b1);
      }
      if (rescale && j > 0) {
        // O holds PV(j-1) relative to r_prev: scale it to r_j once PV(j-1) is
        // done; PV(j) waits for this warpgroup's arrive below
        const float alpha = fast_exp2(r_prev - r_j);
        if (!__all_sync(0xffffffffu, mbar_wait(bar(VEMPTY + (b ^ 1)), ((j - 1) >> 1) & 1,
                                               a, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + 32 * ch, o);
          tmem_ld_wait();
          const uint64_t al2 = f2pack(alpha, alpha);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float x0, x1;
            f2unpack(fmul2(f2pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), al2), x0, x1);
            o[i] = __float_as_uint(x0);
            o[i + 1] = __float_as_uint(x1);
          }
          tmem_st32(lane_base + kColO + 32 * ch, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      if ((threadIdx.x & 127) == 0) DKV_TR(7, j);
      mbar_arrive(bar(PFULL + b));
    }
    // epilogue: wait for the last PV, combine the two warpgroups' row sums at
    // the final reference (the largest, references never decrease), write O
    if (ok && nt > 0) {
      const int jl = nt - 1;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar(VEMPTY + (jl & 1)), (jl >> 1) & 1, a, abort_flag));
    }
    if (ok) {
      lsum[h * 128 + lr] = l;
      lsum[256 + h * 128 + lr] = r_w;
      mbar_arrive(bar(LSUM));
      ok = __all_sync(0xffffffffu, mbar_wait(bar(LSUM), 0, a, abort_flag));
    }
    if (ok && warp_rows) {
      tc_fence_after();
      const float lo = lsum[(h ^ 1) * 128 + lr], ro = lsum[256 + (h ^ 1) * 128 + lr];
      const float rf = fmaxf(r_w, ro);
      // a warpgroup without tiles has l = 0 and reference -inf: weight 2^-inf = 0
      const float lt = l * fast_exp2(r_w - rf) + lo * fast_exp2(ro - rf);
      const float inv = 1.f / lt;
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t o[32];
        tmem_ld32(lane_base + kColO + 64 * h + 32 * ch, o);
        tmem_ld_wait();
        const int col = 64 * h + 32 * ch;
        if (!row_ok) {
          // padding row: nothing to write
        } else if (a.final_out) {
          uint4* dst = reinterpret_cast<uint4*>(a.out + (size_t(u) * cv.rows + r) * kHeadDim + col);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // O column kpos<VB>(c) holds channel c (the V tile's order)
              const __nv_bfloat162 v = __floats2bfloat162_rn(
                  __uint_as_float(o[kpos<VB>(8 * i + 2 * k)]) * inv,
                  __uint_as_float(o[kpos<VB>(8 * i + 2 * k + 1)]) * inv);
              w[k] = *reinterpret_cast<const uint32_t*>(&v);
            }
            dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          // the split's output divided by its row sum, in fp16
          uint4* dst = reinterpret_cast<uint4*>(
              a.part_o + ((size_t(u) * a.part_stride + a.part_base + sp) * cv.rows + r) * kHeadDim + col);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              w[k] = pack_h2(__uint_as_float(o[kpos<VB>(8 * i + 2 * k)]) * inv,
                             __uint_as_float(o[kpos<VB>(8 * i + 2 * k + 1)]) * inv);
            dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (!a.final_out && row_ok && h == 0)
        a.part_ml[(size_t(u) * a.part_stride + a.part_base + sp) * cv.rows + r] = make_float2(rf, lt);
    }
  } else if (warp < 24) {
    regs_dec<kRegProducer>();
    if (warp < 16)
      k_producer_loop<KB, VB, kStages>(a, uls, u, t_begin, nt, pipe, abort_flag, threadIdx.x - 256);
    else
      v_producer_loop<KB, VB, SINK, kStages>(a, uls, u, t_begin, nt, pipe, abort_flag,
                                             threadIdx.x - 512);
  } else {
    regs_dec<kRegControl>();
    if (warp == kLoadWarp) {
      loader_loop<KB, VB, kStages>(a, uls, u, t_begin, nt, pipe, abort_flag, lane);
    } else if (warp == kMmaWarp && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = mbar_wait(bar(QREADY), 0, a, abort_flag);
    tc_fence_after();
    // A fixed order: QK(0), QK(1), then for each tile j QK(j+2) and PV(j).
    // QK(j+2) needs K_(j+2) (KFULL) and S_(j mod 2) read out by the softmax
    // of tile j (SFREE, before P_j is complete); PV(j) needs P_j (PFULL) and
    // V_j (VFULL).  MMAs run in issue order, so when the softmax of tile j
    // starts (QK(j) complete), PV(j-3) and every earlier PV are complete:
    // its parity waits on VEMPTY for PV(j-1) and PV(j-2) cannot match an
    // older phase.  The QK's commit on SFULL also frees its K buffer for the
    // K producers.
    // operand descriptors, computed once: a K-step adds a fixed offset to the
    // start-address field (address / 16, 14 bits; shared memory stays below
    // 256 KB, so the field never carries)
    const uint64_t dq = sdesc_sw128(sm_base + Smem::kQ, 16, 1024);
    const uint64_t dk0 = sdesc_sw128(sm_base + Smem::kK0, 1024, 2048);
    const uint64_t dk1 = sdesc_sw128(sm_base + Smem::kK1, 1024, 2048);
    const uint64_t dv0 = sdesc_sw128(sm_base + Smem::kV0, 1024, 2048);
    const uint64_t dv1 = sdesc_sw128(sm_base + Smem::kV1, 1024, 2048);
    auto issue_qk = [&](int q) {
      DKV_TR(5, q);
      tc_fence_after();
      const int b = q & 1;
      const uint64_t db = b ? dk1 : dk0;
      const uint32_t d_s = tmem + (b ? kColS1 : kColS0);
      // channels 16kk .. 16kk + 15: Q half kk / 4 (16 KB apart), 32 bytes into
      // its 128-byte rows; K tile rows 16kk.. (4 KB per 16 channels)
      mma8_ss(d_s, dq, db, 0u);
      mma_commit(bar(SFULL + b));
      DKV_TR(14, q);
    };
    auto issue_pv = [&](int p) {
      tc_fence_after();
      DKV_TR(8, p);
      const int bb = p & 1;
      const uint64_t dv = bb ? dv1 : dv0;
      const uint32_t a_p = tmem + (bb ? kColP1 : kColP0);
      const int64_t pv_start = (t_begin + p) * TT;
      const int n_tok = uls->n_tok;
      const uint32_t acc0 = p > 0 ? 1u : 0u;
      // tokens 16kk..16kk+15: packed P columns 8kk..8kk+7, V rows 16kk.. (4 KB)
      if (n_tok - pv_start >= TT) {
        mma8_ts(tmem + kColO, a_p, dv, acc0);
      } else {
        const int nk = int(n_tok - pv_start) >> 4;  // the last tile stops at its last token
#pragma unroll 1
        for (int kk = 0; kk < nk; ++kk)
          mma_ts(tmem + kColO, a_p + 8 * kk, dv + uint64_t(256 * kk), kk > 0 ? 1u : acc0);
      }
      mma_commit(bar(VEMPTY + bb));
      DKV_TR(13, p);
    };
#pragma unroll 1
    for (int q = 0; ok && q < 2 && q < nt; ++q) {
      ok = mbar_wait_fast(bar(KFULL + q), 0, a, abort_flag);
      if (ok) issue_qk(q);
    }
#pragma unroll 1
    for (int j = 0; ok && j < nt; ++j) {
      const int q = j + 2;
      if (q < nt) {
        ok = mbar_wait_fast(bar(SFREE + (q & 1)), (j >> 1) & 1, a, abort_flag) &&
             mbar_wait_fast(bar(KFULL + (q & 1)), (q >> 1) & 1, a, abort_flag);
        if (!ok) break;
        issue_qk(q);
      }
      ok = mbar_wait_fast(bar(PFULL + (j & 1)), (j >> 1) & 1, a, abort_flag) &&
           mbar_wait_fast(bar(VFULL + (j & 1)), (j >> 1) & 1, a, abort_flag);
      if (!ok) break;
      issue_pv(j);
    }
    // drain: every MMA issued above completes before TMEM is released
    mma_commit(bar(DONE));
    mbar_wait(bar(DONE), 0, a, abort_flag, /*drain=*/true);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) DKV_TR(10, 0);
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}


// ------------------------------------------------------------ tokens on lanes

// Query groups of 32 rows (one query head per kv-head and 32-token blocks).
// The scores are computed transposed, S^T = K_hat Q^T, so the 128 tokens of
// a tile sit on the 128 TMEM lanes and all four warps of the softmax
// warpgroup work (thread = token, 32 scores per thread), and O^T = V_hat^T P^T
// accumulates with the channels on the lanes.  Both MMAs are M = 128, N = 64
// (the 32 query rows zero-padded; every operand MN-major, 128-byte swizzle):
//   S^T[token][row] += K_hat tile (A: tokens x channels, as dequantized) *
//                      Q^T (B: channels x rows, staged once)
//   O^T[chan][row]  += V_hat^T (A: channels x tokens, the V tile as
//                      dequantized) * P^T (B: tokens x rows, written by the
//                      softmax threads)
// The producers, the loader and the ring are the row-block kernel's.  Each
// row keeps a reference max in registers (the same in every thread), raised
// only when a tile's score exceeds it by more than 8 (log2 units), as in the
// row-block kernel; raising takes a 128-thread reduction and rescales O and
// the per-thread partial row sums.  Per-thread partial row sums (one per
// row) are reduced once at the end.
// Warps: 0-3 softmax, 4-11 K producers, 12-19 V producers, 21 TMEM and MMA
// lane, 22 loader (20, 23 idle); one CTA per SM.
namespace tl {
constexpr int kWarps = 24;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 32;  // query rows per unit
constexpr int kN = 64;     // MMA N (rows padded)
constexpr int kMmaWarp = 21, kLoadWarp = 22;
constexpr int kStages = 2;
// TMEM: four score buffers (tile j uses S_(j mod 4)) and O^T
constexpr int kSBufs = 4;
constexpr uint32_t kColS0 = 0, kColO = 256, kTmemCols = 512;
// D f32, A and B f16, both MN-major, M = 128, N = 64
constexpr uint32_t kIdesc = (1u << 4) | (1u << 15) | (1u << 16) | ((uint32_t(kN) >> 3) << 17) |
                            ((128u >> 4) << 24);
// launch: 80 registers x 768 threads = 61440; softmax 152 x 128, producers
// 64 x 512, control 56 x 128 = 59392
constexpr int kRegSoftmax = 152, kRegProducer = 64, kRegControl = 56;

struct Smem {
  static constexpr uint32_t kK0 = 0, kV0 = 2 * kTileBytes;
  static constexpr uint32_t kP = 4 * kTileBytes;                   // 2 P^T tiles [128 tokens][64 rows]
  static constexpr uint32_t kQ = kP + 2 * 128 * kN * 2;            // Q^T [128 channels][64 rows]
  static constexpr uint32_t kRing = kQ + 128 * kN * 2;
  static constexpr uint32_t kBar = kRing + kStages * ::dkv::kMaxStageBytes;  // 32 mbarriers
  static constexpr uint32_t kFlag = kBar + 32 * 8;                 // [2][4] raise votes
  static constexpr uint32_t kRed = kFlag + 64;                     // [3][4 warps][32 rows] floats
  static constexpr uint32_t kMisc = kRed + 3 * 4 * kRows * 4;      // tmem, abort, lengths
  static constexpr uint32_t kBytes = kMisc + 32;
};
// (VOTE, RED, EPI: the softmax threads' exchanges, bounded waits like every
// other hand-off, so a CTA that aborts cannot leave a thread waiting)
enum Bar {
  KFULL = 0, KEMPTY = 2, VFULL = 4, VEMPTY = 6, SFULL = 8, SFREE = 12, PFULL = 16, QREADY = 18,
  DONE = 19, VOTE = 20, RED = 21, EPI = 22, RFULL = 23, REMPTY = RFULL + kStages
};

// the 16-byte chunk of rows 8k..8k+7 of token / channel t in a [128][64]
// MN-major tile (one 64-element atom per 8 tokens: atom t/8 at (t/8) * 1024)
__device__ __forceinline__ uint32_t nt_off(int t, int k) {
  return uint32_t((t >> 3) * 1024 + (t & 7) * 128 + ((k ^ (t & 7)) << 4));
}

// max over the 32 lanes of every one of the 32 values v[i], the result for
// i = lane returned (a butterfly that halves the values held at each step)
__device__ __forceinline__ float transpose_max(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      // keep rows i (lane bit clear) or i + o (set); send the other
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
    }
  }
  return v[0];  // row = lane
}
__device__ __forceinline__ float transpose_sum(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

// channel of O^T's lane p: the V tile holds its channels in kpos<VB> order
template <int VB>
__device__ __forceinline__ int kpos_inv(int p) {
  for (int t = p & ~15; t < (p & ~15) + 16; ++t)
    if (kpos<VB>(t) == p) return t;
  return p;
}
}  // namespace tl

template <int KB, int VB, bool SINK>
__global__ void __launch_bounds__(tl::kThreads, 1) attn_tl_kernel(const __grid_constant__ AttnArgs a) {
  using S = tl::Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sm_base = smem_u32(sm);
  const uint32_t bar0 = sm_base + S::kBar;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + S::kMisc + 4);

  const CacheView& cv = a.c;
  const int u = blockIdx.x / a.nsplit;
  const int sp = blockIdx.x % a.nsplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const UnitLen ul = unit_len(a, u);
  const int64_t n_tiles = (ul.n_tok + TT - 1) / TT;
  const int64_t t_begin = int64_t(sp) * a.tiles_per_split;
  const int64_t t_end = t_begin + a.tiles_per_split < n_tiles ? t_begin + a.tiles_per_split : n_tiles;
  const int nt = t_end > t_begin ? int(t_end - t_begin) : 0;
  if (nt == 0) {
    // a split past the end of a shorter sequence: an empty partial
    pdl_wait();
    pdl_trigger();
    if (!a.final_out) {
      const size_t prow = (size_t(u) * a.part_stride + a.part_base + sp) * tl::kRows;
      for (int i = threadIdx.x; i < tl::kRows * (kHeadDim / 8); i += tl::kThreads)
        reinterpret_cast<uint4*>(a.part_o + prow * kHeadDim)[i] = make_uint4(0u, 0u, 0u, 0u);
      for (int i = threadIdx.x; i < tl::kRows; i += tl::kThreads)
        a.part_ml[prow + i] = make_float2(-__int_as_float(0x7f800000), 0.f);
    }
    return;
  }
  const UnitLen* uls = reinterpret_cast<const UnitLen*>(sm + S::kMisc + 16);
  const Pipe pipe{sm, sm_base, S::kRing, S::kK0, S::kV0, bar(tl::KFULL), bar(tl::KEMPTY),
                  bar(tl::VFULL), bar(tl::VEMPTY), bar(tl::RFULL), bar(tl::REMPTY)};
  if (threadIdx.x == 0) {
    *reinterpret_cast<UnitLen*>(sm + S::kMisc + 16) = ul;
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(tl::KFULL + b), 256);
      mbar_init(bar(tl::KEMPTY + b), 1);
      mbar_init(bar(tl::VFULL + b), 256);
      mbar_init(bar(tl::VEMPTY + b), 1);
      mbar_init(bar(tl::PFULL + b), 128);
    }
    for (int b = 0; b < tl::kSBufs; ++b) {
      mbar_init(bar(tl::SFULL + b), 1);
      mbar_init(bar(tl::SFREE + b), 128);
    }
    mbar_init(bar(tl::QREADY), 128);
    mbar_init(bar(tl::DONE), 1);
    mbar_init(bar(tl::VOTE), 128);
    mbar_init(bar(tl::RED), 128);
    mbar_init(bar(tl::EPI), 128);
    for (int st = 0; st < tl::kStages; ++st) {
      mbar_init(bar(tl::RFULL + st), 1);
      mbar_init(bar(tl::REMPTY + st), 512);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == tl::kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(tl::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  pdl_wait();  // no global memory access above this line
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) DKV_TR(9, 0);
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------------------ softmax
    regs_inc<tl::kRegSoftmax>();
    const int l = threadIdx.x;  // TMEM lane: token of a tile, then channel of O^T
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    float* red = reinterpret_cast<float*>(sm + S::kRed);     // [3][4][32]
    int* flag = reinterpret_cast<int*>(sm + S::kFlag);         // [2][4]
    const bool qneg = a.scale_log2 < 0.f;
    const float sc = fmaxf(fabsf(a.scale_log2), 1e-30f);
    {
      // Q^T into shared memory: thread = channel l, its 32 rows (bf16 ->
      // fp16, the sign of a negative scale folded in); rows 32..63 zero.  The
      // P^T tile's rows 32..63 (never written again) are zeroed too.
      uint32_t q2[16];
      const uint16_t* qc = a.q + size_t(u) * tl::kRows * kHeadDim + l;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float lo = __uint_as_float(uint32_t(__ldg(qc + size_t(2 * i) * kHeadDim)) << 16);
        const float hi = __uint_as_float(uint32_t(__ldg(qc + size_t(2 * i + 1) * kHeadDim)) << 16);
        q2[i] = pack_h2(qneg ? -lo : lo, qneg ? -hi : hi);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        *reinterpret_cast<uint4*>(sm + S::kQ + tl::nt_off(l, k)) =
            make_uint4(q2[4 * k], q2[4 * k + 1], q2[4 * k + 2], q2[4 * k + 3]);
#pragma unroll
      for (int k = 4; k < 8; ++k) {
        *reinterpret_cast<uint4*>(sm + S::kQ + tl::nt_off(l, k)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(sm + S::kP + tl::nt_off(l, k)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(sm + S::kP + 16384 + tl::nt_off(l, k)) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_async_smem();
      mbar_arrive(bar(tl::QREADY));
    }
    float ref[tl::kRows];    // reference max per row (log2 units), the same in every thread
    float lsum[tl::kRows];   // this thread's (token's) share of each row sum, relative to ref
#pragma unroll
    for (int i = 0; i < tl::kRows; ++i) {
      ref[i] = -__int_as_float(0x7f800000);
      lsum[i] = 0.f;
    }
    bool ok = true;
    int n_raise = 0;  // phases of the tl::RED barrier used so far
#pragma unroll 1
    for (int j = 0; j < nt && ok; ++j) {
      const int b = j & 1;               // vote slot, P buffer
      const int bs = j % tl::kSBufs;     // score buffer (its (j / 4)-th use)
      // tcgen05.ld is warp-collective: every branch around it is warp-uniform
      if (!__all_sync(0xffffffffu, mbar_wait(bar(tl::SFULL + bs), (j / tl::kSBufs) & 1, a, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (threadIdx.x == 0) DKV_TR(6, j);
      const uint32_t s_col = lane_base + tl::kColS0 + 64u * uint32_t(bs);
      float x[tl::kRows];
      auto load_scores = [&]() {
        uint32_t sv[32];
        tmem_ld32(s_col, sv);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < tl::kRows; ++i) x[i] = __uint_as_float(sv[i]) * sc;
      };
      load_scores();
      const int64_t tile_start = (t_begin + j) * TT;
      const int n_tok = uls->n_tok;
      const bool valid = tile_start + l < n_tok;  // (past-the-end tokens have zero K and V)
      // raise the reference where a score exceeds it by more than 8
      bool raise = false;
      if (valid)
#pragma unroll
        for (int i = 0; i < tl::kRows; ++i) raise |= x[i] > ref[i] + 8.f;
      raise = __any_sync(0xffffffffu, raise);
      if (lane == 0) flag[b * 4 + warp] = raise;
      mbar_arrive(bar(tl::VOTE));
      if (!__all_sync(0xffffffffu, mbar_wait(bar(tl::VOTE), j & 1, a, abort_flag))) {
        ok = false;
        break;
      }
      if (threadIdx.x == 0) DKV_TR(12, j);
      raise = flag[b * 4] | flag[b * 4 + 1] | flag[b * 4 + 2] | flag[b * 4 + 3];
      if (raise) {
        // tile max of every row over the 128 tokens (the reduction takes x
        // apart; the scores are read again from tensor memory after it)
        if (!valid)
#pragma unroll
          for (int i = 0; i < tl::kRows; ++i) x[i] = -__int_as_float(0x7f800000);
        red[(b * 4 + warp) * tl::kRows + lane] = tl::transpose_max(x, lane);
        mbar_arrive(bar(tl::RED));
        if (!__all_sync(0xffffffffu, mbar_wait(bar(tl::RED), n_raise & 1, a, abort_flag))) {
          ok = false;
          break;
        }
        ++n_raise;
        float alpha[tl::kRows];
#pragma unroll
        for (int i = 0; i < tl::kRows; ++i) {
          const float* rr = red + b * 4 * tl::kRows + i;
          const float tm = fmaxf(fmaxf(rr[0], rr[tl::kRows]), fmaxf(rr[2 * tl::kRows], rr[3 * tl::kRows]));
          const float nr = tm > ref[i] + 8.f ? fmaxf(ref[i], tm) : ref[i];
          alpha[i] = fast_exp2(ref[i] - nr);  // 1 when unchanged, 0 from -inf
          ref[i] = nr;
          lsum[i] *= alpha[i];
        }
        if (j > 0) {
          // O^T holds PV up to tile j-1 relative to the old references: scale
          // its row columns once that PV has completed
          if (!__all_sync(0xffffffffu, mbar_wait(bar(tl::VEMPTY + ((j - 1) & 1)), ((j - 1) >> 1) & 1, a,
                                                 abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t o[16];
            tmem_ld16(lane_base + tl::kColO + 16 * h, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[16 * h + i]);
            tmem_st16(lane_base + tl::kColO + 16 * h, o);
          }
          tmem_st_wait();
        }
        load_scores();
      }
      // P = 2^(x - ref) (0 past the end), fp16 pairs; row sums in fp32
      uint32_t pk[tl::kRows / 2];
#pragma unroll
      for (int i = 0; i < tl::kRows; i += 2) {
        const float p0 = valid ? fast_exp2(x[i] - ref[i]) : 0.f;
        const float p1 = valid ? fast_exp2(x[i + 1] - ref[i + 1]) : 0.f;
        lsum[i] += p0;
        lsum[i + 1] += p1;
        pk[i / 2] = pack_h2(p0, p1);
      }
      // P^T buffer b is free once PV(j-2) has completed
      if (j > 1 && !__all_sync(0xffffffffu, mbar_wait(bar(tl::VEMPTY + b), ((j - 2) >> 1) & 1, a,
                                                      abort_flag))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        *reinterpret_cast<uint4*>(sm + S::kP + 16384u * uint32_t(b) + tl::nt_off(l, k)) =
            make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
      fence_async_smem();
      tc_fence_before();
      if (threadIdx.x == 0) DKV_TR(7, j);
      mbar_arrive(bar(tl::PFULL + b));
      mbar_arrive(bar(tl::SFREE + bs));  // (S_bs was last read above)
    }
    // epilogue: row sums over the 128 tokens, then O^T / l per row
    if (ok) {
      const int jl = nt - 1;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar(tl::VEMPTY + (jl & 1)), (jl >> 1) & 1, a, abort_flag));
    }
    if (ok) {
      float* rs = red + 2 * 4 * tl::kRows;  // (the raise path's halves stay untouched)
      rs[warp * tl::kRows + lane] = tl::transpose_sum(lsum, lane);
      mbar_arrive(bar(tl::EPI));
      ok = __all_sync(0xffffffffu, mbar_wait(bar(tl::EPI), 0, a, abort_flag));
    }
    if (ok) {
      const float* rs = red + 2 * 4 * tl::kRows;
      tc_fence_after();
      uint32_t o[32];
      tmem_ld32(lane_base + tl::kColO, o);
      tmem_ld_wait();
      const int ch = tl::kpos_inv<VB>(l);  // O^T lane l holds channel kpos^-1(l)
#pragma unroll
      for (int i = 0; i < tl::kRows; ++i) {
        const float lt = (rs[i] + rs[tl::kRows + i]) + (rs[2 * tl::kRows + i] + rs[3 * tl::kRows + i]);
        const float ov = __uint_as_float(o[i]);
        if (a.final_out) {
          const __nv_bfloat16 v = __float2bfloat16_rn(ov / lt);
          a.out[(size_t(u) * tl::kRows + i) * kHeadDim + ch] = *reinterpret_cast<const uint16_t*>(&v);
        } else {
          const size_t prow = (size_t(u) * a.part_stride + a.part_base + sp) * tl::kRows + i;
          a.part_o[prow * kHeadDim + ch] = __float2half_rn(ov / lt);
          if (l == 0) a.part_ml[prow] = make_float2(ref[i], lt);
        }
      }
    }
  } else if (warp < 20) {
    regs_dec<tl::kRegProducer>();
    if (warp < 12)
      k_producer_loop<KB, VB, tl::kStages>(a, uls, u, t_begin, nt, pipe, abort_flag, threadIdx.x - 128);
    else
      v_producer_loop<KB, VB, SINK, tl::kStages>(a, uls, u, t_begin, nt, pipe, abort_flag,
                                             threadIdx.x - 384);
  } else {
    regs_dec<tl::kRegControl>();
    if (warp == tl::kLoadWarp) {
      loader_loop<KB, VB, tl::kStages>(a, uls, u, t_begin, nt, pipe, abort_flag, lane);
    } else if (warp == tl::kMmaWarp && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      // QK(j) needs K_j and S_(j mod 4) read (SFREE of tile j-4); PV(j) needs
      // P_j (PFULL of buffer j mod 2) and V_j.  QK runs up to three tiles ahead of PV.
      bool ok = mbar_wait(bar(tl::QREADY), 0, a, abort_flag);
      tc_fence_after();
      const uint32_t qbase = sm_base + S::kQ;
      int nq = 0, np = 0;
      auto issue_qk = [&]() {
        tc_fence_after();
        DKV_TR(5, nq);
        const int b = nq & 1, bs = nq % tl::kSBufs;
        const uint32_t kbase = sm_base + S::kK0 + b * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // channels 16kk .. 16kk + 15
          asm volatile(
              "{\n\t.reg .pred p;\n\t"
              "setp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(
                  tmem + tl::kColS0 + 64u * uint32_t(bs)),
              "l"(sdesc_sw128(kbase + 4096 * kk, 1024, 2048)), "l"(sdesc_sw128(qbase + 2048 * kk, 8192, 1024)),
              "r"(tl::kIdesc), "r"(kk > 0 ? 1u : 0u)
              : "memory");
        mma_commit(bar(tl::KEMPTY + b));
        mma_commit(bar(tl::SFULL + bs));
        ++nq;
      };
#pragma unroll 1
      while (ok && np < nt) {
        // issue every QK that is ready and allowed (at most one ahead of PV)
        auto s_free = [&](bool wait) {  // S_(nq mod 4) read by the softmax of tile nq - 4
          if (nq < tl::kSBufs) return true;
          const uint32_t sb = bar(tl::SFREE + nq % tl::kSBufs);
          const uint32_t ph = ((nq - tl::kSBufs) / tl::kSBufs) & 1;
          return wait ? mbar_wait(sb, ph, a, abort_flag) : mbar_test(sb, ph);
        };
        while (nq < nt && nq <= np + tl::kSBufs - 1 &&
               mbar_test(bar(tl::KFULL + (nq & 1)), (nq >> 1) & 1) && s_free(false))
          issue_qk();
        if (np == nq) {
          ok = mbar_wait(bar(tl::KFULL + (nq & 1)), (nq >> 1) & 1, a, abort_flag) && s_free(true);
          if (ok) issue_qk();
          continue;
        }
        const int bb = np & 1;
        if (!mbar_wait(bar(tl::PFULL + bb), (np >> 1) & 1, a, abort_flag) ||
            !mbar_wait(bar(tl::VFULL + bb), (np >> 1) & 1, a, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        DKV_TR(8, np);
        const uint32_t vbase = sm_base + S::kV0 + bb * kTileBytes;
        const uint32_t pbase = sm_base + S::kP + 16384u * uint32_t(bb);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // tokens 16kk .. 16kk + 15
          asm volatile(
              "{\n\t.reg .pred p;\n\t"
              "setp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem + tl::kColO),
              "l"(sdesc_sw128(vbase + 4096 * kk, 1024, 2048)), "l"(sdesc_sw128(pbase + 2048 * kk, 8192, 1024)),
              "r"(tl::kIdesc), "r"((np > 0 || kk > 0) ? 1u : 0u)
              : "memory");
        mma_commit(bar(tl::VEMPTY + bb));
        ++np;
      }
      // drain: every MMA issued above completes before TMEM is released
      mma_commit(bar(tl::DONE));
      mbar_wait(bar(tl::DONE), 0, a, abort_flag, /*drain=*/true);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) DKV_TR(10, 0);
  if (warp == tl::kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tl::kTmemCols));
  }
}

template <int KB, int VB, bool SINK>
cudaError_t launch_tl(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = tl::Smem::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tl_kernel<KB, VB, SINK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(attn_tl_kernel<KB, VB, SINK>, dim3(unsigned(a.c.U) * unsigned(a.nsplit)),
                 dim3(tl::kThreads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int KB, int VB, bool SINK>
cudaError_t launch_kvs(const AttnArgs& a, cudaStream_t s) {
  if (a.tc_layout == 1) return launch_tl<KB, VB, SINK>(a, s);
  const size_t smem = SmemTail<KB, VB>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<KB, VB, SINK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const unsigned nrb = unsigned((a.c.rows + 127) / 128);
  e = launch_pdl(attn_tc_kernel<KB, VB, SINK>, dim3(unsigned(a.c.U) * unsigned(a.nsplit) * nrb),
                 dim3(kThreads), smem, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// caches with a sink (and quantized V) run the instantiation that reads the
// sink's bf16 V rows; the others the one without that check
template <int KB, int VB>
cudaError_t launch_kv(const AttnArgs& a, cudaStream_t s) {
  if (VB < 16 && a.c.sink > 0) return launch_kvs<KB, VB, true>(a, s);
  return launch_kvs<KB, VB, false>(a, s);
}

template <int KB>
cudaError_t launch_k(const AttnArgs& a, cudaStream_t s) {
  switch (a.c.vb) {
    case 2: return launch_kv<KB, 2>(a, s);
    case 3: return launch_kv<KB, 3>(a, s);
    case 4: return launch_kv<KB, 4>(a, s);
    default: return launch_kv<KB, 16>(a, s);
  }
}

}  // namespace

// any query group of 32..256 rows (a multiple of 32): M = 128 per row block
bool tc_supported(const CacheView& c) {
  return c.d == kHeadDim && c.rows >= 32 && c.rows <= 256 && c.rows % 32 == 0;
}

cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t s) {
  if (!tc_supported(a.c)) return cudaErrorNotSupported;
  switch (a.c.kb) {
    case 2: return launch_k<2>(a, s);
    case 3: return launch_k<3>(a, s);
    case 4: return launch_k<4>(a, s);
    default: return launch_k<16>(a, s);
  }
}

}  // namespace dkv

#ifdef DKV_TRACE
// trace build only: the stamps of the last traced launch (16 x 64 uint64, host
// buffer), and their reset to zero
extern "C" int dkv_trace_read(unsigned long long* out) {
  return int(cudaMemcpyFromSymbol(out, dkv::g_trace, sizeof(dkv::g_trace)));
}
extern "C" int dkv_trace_clear(void) {
  static unsigned long long zero[16][64] = {};
  return int(cudaMemcpyToSymbol(dkv::g_trace, zero, sizeof(zero)));
}
#endif
