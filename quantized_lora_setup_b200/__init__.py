"""B200-native NF4 pass: blockwise NF4 quantization, double quantization, per-layer
reconstruction error and top-K selection under a byte budget (the AQLoRA setup pass),
plus standalone NF4 dequantization.

The compute lives in ``libaqnf4.so`` (CUDA, sm_100a), whose C ABI is declared in
``include/aqnf4.h``; :mod:`quantized_lora_setup_b200.aqnf4` binds it.  Importing this
package does not load the library; the first call into the binding does, and fails
loudly if it was not built.
"""
__all__ = ["aqnf4", "synth", "build"]
