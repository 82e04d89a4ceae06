"""B200-native mLSTM cell forward and decode step.

The compute path is the C-ABI library ``libxlstm_mlstm.so`` (hand-written
sm_100a CUDA kernels); ``binding`` marshals arguments into it and does no
arithmetic of its own.  ``synthetic`` draws seeded inputs.  Importing this
package loads nothing; ``binding.load()`` loads the library and fails loudly
if it is missing.
"""
__all__ = ["binding", "synthetic"]
