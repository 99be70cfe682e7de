"""B200-native forward pass of a gpt-oss-style sparse MoE layer with MXFP4 experts.

The compute path is the C-ABI shared library built from ``csrc/`` (hand-written
sm_100a CUDA). ``binding`` is a thin ctypes layer over it; ``workloads`` draws
the seeded synthetic inputs. Nothing is imported eagerly so that the input
generator can be used without loading the CUDA library.
"""

__all__ = ["binding", "workloads"]
