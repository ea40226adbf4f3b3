// Primary-only KV append ("Sintesi Tecnica: Dual-Flow Transformers", section
// "Architettura Core": only the primary flow writes the persistent cache).
// One CTA per sequence copies its Hkv new K rows and V rows into the page slot
// of position positions[b] with 16-byte vector stores: a bit-exact copy.
#include "common.cuh"
#include "host_util.h"

namespace df {
namespace append {

struct Params {
  const uint8_t* k_new;
  const uint8_t* v_new;
  int64_t new_stride_bytes;
  uint8_t* k_cache;
  uint8_t* v_cache;
  const int32_t* block_table;
  int max_blocks_per_seq;
  const int32_t* positions;
  int Hkv;
  int row_bytes;  // D * element size
  int block_size;
  int num_blocks;
  int32_t* err;
};

__global__ void __launch_bounds__(256) kv_append_kernel(const Params p) {
  const int b = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  const int pos = p.positions[b];
  if (pos < 0 || pos / p.block_size >= p.max_blocks_per_seq) {
    if (threadIdx.x == 0) set_err(p.err, DF_DEVERR_POSITION);
    return;
  }
  const int page = p.block_table[static_cast<int64_t>(b) * p.max_blocks_per_seq + pos / p.block_size];
  if (page < 0 || page >= p.num_blocks) {
    if (threadIdx.x == 0) set_err(p.err, DF_DEVERR_BLOCK);
    return;
  }
  const int slot = pos % p.block_size;
  const int vec_per_row = p.row_bytes / 16;
  const int nvec = p.Hkv * vec_per_row;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    const int g = v / vec_per_row, off = (v % vec_per_row) * 16;
    const int64_t src = static_cast<int64_t>(b) * p.new_stride_bytes +
                        static_cast<int64_t>(g) * p.row_bytes + off;
    const int64_t dst =
        ((static_cast<int64_t>(page) * p.Hkv + g) * p.block_size + slot) * p.row_bytes + off;
    *reinterpret_cast<uint4*>(p.k_cache + dst) = *reinterpret_cast<const uint4*>(p.k_new + src);
    *reinterpret_cast<uint4*>(p.v_cache + dst) = *reinterpret_cast<const uint4*>(p.v_new + src);
  }
}

}  // namespace append
}  // namespace df

extern "C" df_status dualflow_kv_append(const void* k_new, const void* v_new, int64_t new_stride_b,
                                        void* k_cache, void* v_cache, const int32_t* block_table,
                                        int max_blocks_per_seq, const int32_t* positions, int B,
                                        int Hkv, int D, int block_size, int num_blocks, int dtype,
                                        int32_t* err_flag, void* stream) {
  using namespace df;
  if (!k_new || !v_new || !k_cache || !v_cache || !block_table || !positions) return DF_ERR_NULL;
  if (B < 1 || Hkv < 1 || D < 1 || block_size < 1 || num_blocks < 1 || max_blocks_per_seq < 1)
    return DF_ERR_SHAPE;
  if (B > 2147483647 / 2) return DF_ERR_SHAPE;
  if (dtype != DF_FP32 && dtype != DF_BF16) return DF_ERR_UNSUPPORTED;
  const int esize = dtype == DF_BF16 ? 2 : 4;
  const int64_t stride = new_stride_b ? new_stride_b : static_cast<int64_t>(Hkv) * D;
  if (stride < static_cast<int64_t>(Hkv) * D) return DF_ERR_SHAPE;
  if ((D * esize) % 16 != 0 || (stride * esize) % 16 != 0) return DF_ERR_ALIGN;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return DF_ERR_ALIGN;
  append::Params p;
  p.k_new = static_cast<const uint8_t*>(k_new);
  p.v_new = static_cast<const uint8_t*>(v_new);
  p.new_stride_bytes = stride * esize;
  p.k_cache = static_cast<uint8_t*>(k_cache);
  p.v_cache = static_cast<uint8_t*>(v_cache);
  p.block_table = block_table;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.positions = positions;
  p.Hkv = Hkv;
  p.row_bytes = D * esize;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  p.err = err_flag;
  const int nvec = Hkv * (D * esize / 16);
  const int threads = nvec >= 256 ? 256 : ((nvec + 31) / 32) * 32;
  if (launch_pdl(append::kv_append_kernel, dim3(B), dim3(threads), 0,
                 static_cast<cudaStream_t>(stream), p) != cudaSuccess)
    return DF_ERR_CUDA;
  return DF_OK;
}
