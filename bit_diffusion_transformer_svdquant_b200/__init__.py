"""B200 (sm_100a) SVDQuant-style W4A4 + low-rank linear layer.

The layer ("Bringing Nunchaku 4-bit diffusion inference to Diffusers", "SVDQuant deep dive"):
4-bit NVFP4 weights and activations, outliers absorbed by a 16-bit low-rank branch W = L1 L2 + R,
the branch's down-projection fused with activation quantization and its up-projection fused with
the 4-bit GEMM. The compute lives in libsvdq.so (C ABI in include/svdq.h); this package is its thin
Python binding plus the seeded synthetic workloads and an offline weight-preparation helper.
"""
from ._lib import (EPI_BIAS, EPI_BIAS_SWIGLU, EPI_NONE, EPI_SWIGLU, Fp8rAct, Fp8rWeight, PackedWeight,
                   QuantizedAct, SvdqError, calibrate_act, device_status, export_act, export_act_fp8r,
                   export_weight, export_weight_fp8r, gemm, gemm_fp8r, gemm_swiglu_quant, linear, linear_fp8r, mlp,
                   quantize_act,
                   quantize_act_fp8r, set_wait_limit_ns, watchdog_selftest)

__all__ = ["EPI_BIAS", "EPI_BIAS_SWIGLU", "EPI_NONE", "EPI_SWIGLU", "Fp8rAct", "Fp8rWeight", "PackedWeight",
           "QuantizedAct", "SvdqError", "calibrate_act", "device_status", "export_act", "export_act_fp8r",
           "export_weight", "export_weight_fp8r", "gemm", "gemm_fp8r", "gemm_swiglu_quant", "linear", "linear_fp8r",
           "mlp", "quantize_act",
           "quantize_act_fp8r", "set_wait_limit_ns", "watchdog_selftest"]
