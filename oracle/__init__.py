"""Oracle package: CPU reference of the DeepSeekMoE layer (test infrastructure).

Only tests/, the smoke check and the benchmark's CPU-baseline leg use this
package.  It shares no code with the CUDA library and imports nothing from it.
Two independent implementations: moe_ref (plain C++17 + OpenMP in float64,
oracle/moe_ref.cpp, loaded through ctypes) and moe_oracle / moe_backward
(numpy in float64); tests check them against each other and against pins.
"""
from .moe_oracle import *  # noqa: F401,F403
