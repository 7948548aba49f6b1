"""Oracle for the DeepSeekMoE layer forward — TEST INFRASTRUCTURE ONLY.

A plain CPU (C++17, fp64, OpenMP) restatement of the layer, used to check the
CUDA library. Only tests/, the package's smoke() entry and bench.py's CPU
baseline may import it; the product path never does.
"""
