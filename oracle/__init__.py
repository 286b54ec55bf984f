"""fp64 CPU oracle of the LoRA-MLP sub-block and of the 4-bit weight codes.

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline (and its reference arm) may import, call or execute anything here.  The
CUDA product path (lora_fine_tuning_rmsnorm_b200) never imports it and shares no
code with it; the only module both sides use is the seeded input generator
lora_fine_tuning_rmsnorm_b200.synth, which holds none of the method's arithmetic.

Parity status: every function here is pinned by tests/test_oracle_*.py against
finite differences, closed forms, invariants and brute force (no function is
"parity unpinned").
"""
from . import lora_mlp_ref, quant4_ref  # noqa: F401
