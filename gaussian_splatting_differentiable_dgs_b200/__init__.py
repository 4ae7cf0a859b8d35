"""B200-native training step of 3D Gaussian Splatting with the BoundedGS
memory scheme: a C-ABI CUDA library (``libgs.so``) and a thin binding.

Importing the package does not load the CUDA library; ``binding.lib()`` and
the ``Step`` driver do, and fail loudly when it is missing.
"""
__version__ = "0.1.0"
