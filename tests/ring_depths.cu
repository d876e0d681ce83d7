// Test helper (host program): prints the ring depths of every dequantizing instantiation of the fused GEMM, as the
// kernel's own configuration computes them, for the randomized protocol model in test_ring_protocol.py.
// Columns: BN AM KB QS AS BS G acc_bufs.
#include <cstdio>

#include "../qlora_fine_tuning_blockwise_b200/csrc/umma_gemm.cuh"

using namespace qlora;

template <int BN, int AM, int KB, int EPI = EPI_PLAIN>
void row() {
  using C = UmmaCfg<BN, AM, false, KB, false, EPI>;
  std::printf("%d %d %d %d %d %d %d %d\n", BN, AM, KB, C::kQStages, C::kAStages, C::kBStages, C::kDeqGroups,
              C::kAccBufs);
}

int main() {
  row<16, A_DEQ_TMEM, 1>();
  row<32, A_DEQ_TMEM, 1>();
  row<64, A_DEQ_TMEM, 1>();
  row<128, A_DEQ_TMEM, 1>();
  row<256, A_DEQ_TMEM, 1>();
  row<16, A_DEQ_TMEM, 4>();
  row<32, A_DEQ_TMEM, 4>();
  row<64, A_DEQ_TMEM, 4>();
  row<16, A_DEQ_MN, 1>();
  row<32, A_DEQ_MN, 1>();
  row<64, A_DEQ_MN, 1>();
  row<128, A_DEQ_MN, 1>();
  row<256, A_DEQ_MN, 1>();
  row<16, A_DEQ_TMEM_T, 1>();
  row<32, A_DEQ_TMEM_T, 1>();
  row<64, A_DEQ_TMEM_T, 1>();
  row<128, A_DEQ_TMEM_T, 1>();
  row<256, A_DEQ_TMEM_T, 1>();
  row<128, A_DEQ_TMEM, 1, EPI_SWIGLU_FWD>();
  row<256, A_DEQ_TMEM, 1, EPI_SWIGLU_FWD>();
  return 0;
}
