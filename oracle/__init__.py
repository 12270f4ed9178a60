"""CPU oracle for the QLoRA-adapted linear layer (test infrastructure only)."""
from .qlora_oracle import *  # noqa: F401,F403
