// Tensor-parallel grouped-query attention block.
//   "Tensor Parallelism" (klaylearn), Notes, grouped-query paragraph: per shard n_q/p query heads
//   and n_kv/p KV heads (column-parallel Q/K/V), local attention, row-parallel output projection
//   giving a full-width partial, partials summed.
#include "attn.cuh"

extern "C" size_t tp_attn_wqkv_packed_bytes(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  return tp::attn_layout_of(desc, &L) == TP_OK ? L.wqkv_bytes : 0;
}
extern "C" size_t tp_attn_wo_packed_bytes(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  return tp::attn_layout_of(desc, &L) == TP_OK ? L.wo_bytes : 0;
}
extern "C" size_t tp_attn_fwd_workspace(const tp_attn_desc* desc) {
  tp::AttnLayout L;
  return tp::attn_layout_of(desc, &L) == TP_OK ? L.ws_bytes : 0;
}

extern "C" tp_status tp_attn_pack(const tp_attn_desc* desc, const void* wq, const void* wk,
                                  const void* wv, const void* wo, void* wqkv_p, void* wo_p,
                                  void* stream) {
  tp::clear_error();
  tp::AttnLayout L;
  tp_status st = tp::attn_layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (!wq || !wk || !wv || !wo || !wqkv_p || !wo_p)
    return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  return tp::attn_pack(L, wq, wk, wv, wo, wqkv_p, wo_p, static_cast<cudaStream_t>(stream));
}

extern "C" tp_status tp_attn_fwd(const tp_attn_desc* desc, const void* x, const void* wqkv_p,
                                 const void* wo_p, void* k_cache, void* v_cache,
                                 const void* residual, void* y, void* y_norm, void* workspace,
                                 size_t ws_bytes, void* stream) {
  tp::clear_error();
  tp::AttnLayout L;
  tp_status st = tp::attn_layout_of(desc, &L);
  if (st != TP_OK) return st;
  if (desc->reduce_mode == TP_REDUCE_FUSED && !L.tc)
    return tp::set_error(TP_ERR_UNSUPPORTED,
                         "TP_REDUCE_FUSED needs the tensor-core path (bf16, h a multiple of 8)");
  if (L.tokens == 0) {
    tp::count_reduction();
    return TP_OK;
  }
  if (!x || !wqkv_p || !wo_p || !y) return tp::set_error(TP_ERR_INVALID_ARG, "null pointer");
  if (L.kv_len > 0 && (!k_cache || !v_cache))
    return tp::set_error(TP_ERR_INVALID_ARG, "decode needs k_cache and v_cache");
  if (L.kv_len > 0 && ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15))
    return tp::set_error(TP_ERR_INVALID_ARG, "k_cache and v_cache must be 16-byte aligned");
  if (!workspace) return tp::set_error(TP_ERR_INVALID_ARG, "workspace is null");
  if (ws_bytes < L.ws_bytes) return tp::set_error(TP_ERR_WORKSPACE, "workspace too small");
  st = tp::attn_forward(L, x, wqkv_p, wo_p, k_cache, v_cache, residual, y, y_norm, workspace,
                        static_cast<cudaStream_t>(stream));
  if (st == TP_OK) tp::count_reduction();
  return st;
}
