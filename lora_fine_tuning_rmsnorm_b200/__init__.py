"""B200-native (sm_100a) LoRA-augmented Llama MLP sub-block: RMSNorm -> gate/up
(+LoRA) -> SwiGLU -> down (+LoRA), forward and hand-derived backward, behind the
C-ABI library liblora_mlp.so (see include/lora_mlp.h).

The compute entry points live in `lora_fine_tuning_rmsnorm_b200.ops` (ctypes
binding of the C ABI); importing this package does not load the library.
"""
__all__ = ["ops", "synth", "configs"]
