"""B200-native (sm_100a) Ideogram 4 single-stream DiT block hot path.

The compute lives in ``libjab_b200.so`` (C ABI in ``include/jab_dit.h``);
``joint_attention_block_b200.ops`` is the thin Python binding.  Importing the
package does not load the library; the first call does, and fails loudly if
the library has not been built.
"""
from . import _abi as ops  # noqa: F401
from . import synth  # noqa: F401
from . import fp8_checkpoint  # noqa: F401

__all__ = ["ops", "synth", "fp8_checkpoint"]
