"""B200-native FlashBlock block-diffusion attention step.

The CUDA library (libfb.so, C-ABI declared in include/fb.h) does the work;
``block_diffusion_attention_flashblock_b200.fb`` is its thin ctypes binding.
``workloads`` draws seeded synthetic inputs.  Importing the package loads
nothing; the binding loads the library on first use and fails loudly if it is
missing.
"""
__all__ = ["fb", "workloads"]
