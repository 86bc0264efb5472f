"""B200 (sm_100a) BitLinear W1.58A8 forward of BitNet b1.58.

The compute lives in ``libbitlinear.so`` (C ABI, declared in include/bitlinear.h);
:mod:`ternary_weight_bitlinear_b200.bitlinear` is its thin ctypes binding.
"""
from .bitlinear import (BL_MAX_K, BL_OUT_BF16, BL_OUT_F32, BitLinearError, LIB_PATH,  # noqa: F401
                        bitlinear_accumulate, bitlinear_act_quant, bitlinear_device_status,
                        bitlinear_forward, bitlinear_forward_batch,
                        bitlinear_forward_batch_workspace_size, bitlinear_forward_quantized,
                        bitlinear_forward_quantized_batch, bitlinear_forward_gate_up,
                        bitlinear_pack_gate_up, bitlinear_pack_gate_up_workspace_size,
                        bitlinear_forward_online, bitlinear_forward_online_workspace_size,
                        bitlinear_backward_ste, make_chain, bitlinear_decode_chain_prepare,
                        bitlinear_decode_chain_run, bitlinear_decode_chain_workspace_size,
                        make_batch,
                        make_quantized_batch,
                        bitlinear_forward_workspace_size, bitlinear_pack,
                        bitlinear_pack_ternary, bitlinear_pack_workspace_size,
                        bitlinear_quantized_batch_workspace_size,
                        bitlinear_selftest_wait_timeout,
                        bitlinear_relu2_mul, bitlinear_unpack, lib, status_string,
                        bitlinear_rope, bitlinear_attn_decode, bitlinear_attn_decode_workspace_size)
