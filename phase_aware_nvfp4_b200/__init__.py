"""B200-native NVFP4 prefill linear layer (Mix-Quant hot path).

Mix-Quant ("Mix-Quant: Quantized Prefilling, Precise Decoding for Agentic
LLMs", section 3.3) runs the prefill phase with NVFP4 weight-and-activation
quantization and keeps decoding in BF16 on the same base weights.  This
package is the data-parallel core of that prefill phase on sm_100a:

* ``mixquant``   -- thin ctypes binding over ``libmixquant.so`` (the C ABI
  declared in ``include/mixquant.h``); argument marshalling only.
* ``workloads``  -- seeded synthetic inputs shaped like the paper's workloads.
* ``build``      -- nvcc build of the CUDA library for sm_100a.

Importing the package does not load CUDA code; the first call into
``mixquant`` does, and raises if the compiled library is missing.
"""

__all__ = ["mixquant", "workloads"]
__version__ = "0.1.0"
