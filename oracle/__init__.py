"""Oracle package: CPU reference of the DeepSeekMoE layer (test infrastructure).

Only tests/, the smoke check and the benchmark's CPU-baseline leg use this
package.  It shares no code with the CUDA library and imports nothing from it.
"""
from .moe_oracle import *  # noqa: F401,F403
