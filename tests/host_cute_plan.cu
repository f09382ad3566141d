// Host program for tests/test_w4a4_plan_host.py: lets CuTe (the CUTLASS
// layout library, header-only) derive the block-scaled FP4 MMA plan for the
// W4A4 GEMM's configuration -- M = N = 128, a K tile of 256 E2M1 elements,
// UE4M3 scales per 16 -- and prints it beside the kernel's own descriptors
// (csrc/w4a4_desc.cuh) as "key value" lines.  Runs on the host only.
#include <cstdio>

#include <cute/config.hpp>
// plain inline instead of forced inlining on the host (GCC refuses to
// force-inline CuTe's mutually recursive bit rotations)
#undef CUTE_HOST_DEVICE
#define CUTE_HOST_DEVICE inline __host__ __device__
#undef CUTE_HOST
#define CUTE_HOST inline __host__
#include <cute/tensor.hpp>
#include <cute/atom/mma_atom.hpp>
#include <cute/atom/mma_traits_sm100.hpp>
#include <cute/atom/copy_traits_sm100.hpp>
#include <cutlass/detail/sm100_blockscaled_layout.hpp>

#include "w4a4_desc.cuh"

using namespace cute;

int main() {
  using E2M1 = cutlass::float_e2m1_t;
  using UE4M3 = cutlass::float_ue4m3_t;
  using MmaOp = SM100_MMA_MXF4_SS<E2M1, E2M1, float, UE4M3, 128, 128, 16, UMMA::Major::K, UMMA::Major::K>;
  auto tiled_mma = make_tiled_mma(MmaOp{});
  using Tile = Shape<_128, _128, _256>;
  using Cfg = cutlass::detail::Sm1xxBlockScaledConfig<16>;

  // instruction descriptor
  const uint32_t idesc = UMMA::make_instr_desc_block_scaled<E2M1, E2M1, float, UE4M3, 128, 128, UMMA::Major::K,
                                                             UMMA::Major::K>();
  printf("idesc_cute %u\n", idesc);
  printf("idesc_kernel %u\n", bsr::w4gemm::idesc_mxf4(128, 128));

  // shared-memory scale layout: byte offset of (row, scale j, K block kb)
  auto sSFA = Cfg::deduce_smem_layoutSFA(tiled_mma, Tile{});
  for (int kb = 0; kb < 4; ++kb)
    for (int row = 0; row < 128; row += 31)
      for (int j = 0; j < 4; ++j) {
        const int off = sSFA(make_coord(make_coord(make_coord(make_coord(row % 32, row / 32), 0), make_coord(0, j)), 0,
                                        make_coord(0, kb)));
        printf("smem_sf %d %d %d %d\n", row, j, kb, off);
      }

  // tensor-memory scale layout (byte-column addressing: lane << 18 | byte)
  auto tCtSFA = make_tensor<typename decltype(tiled_mma)::FrgTypeSFA>(shape(sSFA));
  for (int kb = 0; kb < 4; ++kb)
    for (int row = 0; row < 128; row += 31)
      for (int rep = 0; rep < 4; ++rep)
        for (int j = 0; j < 4; ++j) {
          const int off = tCtSFA.layout()(make_coord(
              make_coord(make_coord(make_coord(row % 32, row / 32), rep), make_coord(0, j)), 0, make_coord(0, kb)));
          printf("tmem_sf %d %d %d %d %d\n", row, rep, j, kb, off);
        }

  // the tcgen05.cp copies and their source descriptors
  auto sptr = make_smem_ptr(reinterpret_cast<UE4M3*>(0));
  auto tCsSFA = make_tensor(sptr, sSFA);
  auto s_compact = make_tensor(tCsSFA.data(), filter_zeros(tCsSFA.layout()));
  auto t_compact = make_tensor(tCtSFA.data(), filter_zeros(tCtSFA.layout()));
  auto thr = make_utccp_copy(SM100_UTCCP_4x32dp128bit_1cta{}, t_compact).get_slice(0);
  auto src = thr.partition_S(s_compact);
  auto dst = thr.partition_D(t_compact);
  auto desc = get_utccp_smem_desc_tensor<SM100_UTCCP_4x32dp128bit_1cta>(src);
  const int copies = size<3>(desc);
  printf("copies %d\n", copies);
  for (int c = 0; c < copies; ++c) {
    UMMA::SmemDescriptor d;
    d.desc_ = uint64_t(desc(make_coord(0, 0, 0, c)));
    // the kernel's descriptor for the same atom (start address 512 * c)
    UMMA::SmemDescriptor mine;
    mine.desc_ = bsr::w4gemm::smem_desc_k_plain(512u * (uint32_t)c);
    printf("cp_desc %d %llu %llu\n", c, (unsigned long long)d.desc_, (unsigned long long)mine.desc_);
    printf("cp_dst %d %d\n", c, (int)dst.layout()(make_coord(0, 0, 0, c)));
  }

  // operand descriptors of a 128 x 256 E2M1 tile, 128-byte swizzle, K-major
  auto sA_layout = tile_to_shape(UMMA::Layout_K_SW128_Atom<E2M1>{}, make_shape(_128{}, _256{}));
  auto sA = make_tensor(make_smem_ptr(reinterpret_cast<E2M1*>(0)), sA_layout);
  auto tCrA = tiled_mma.make_fragment_A(tiled_mma.get_slice(0).partition_A(sA));
  for (int kb = 0; kb < size<2>(tCrA); ++kb) {
    UMMA::SmemDescriptor d;
    d.desc_ = uint64_t(tCrA(0, 0, kb));
    printf("a_desc %d %u %u %u %u %u\n", kb, (unsigned)d.start_address_, (unsigned)d.leading_byte_offset_,
           (unsigned)d.stride_byte_offset_, (unsigned)d.layout_type_, (unsigned)d.version_);
  }
  return 0;
}
