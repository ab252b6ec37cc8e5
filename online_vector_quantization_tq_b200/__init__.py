"""B200-native TurboQuant-style online vector quantization.

The compute path is the CUDA library libtq.so (C ABI in include/tq.h); this
package exposes it to PyTorch through ``binding`` (ctypes, argument
marshalling only).  Build the library with ``build.build()``.
"""
from .binding import (Encoded, Quantizer, TQError, lib, score_workspace, topk_workspace,  # noqa: F401
                      tq_attend, tq_codebook, tq_codebook_host, tq_codebook_mse, tq_codebook_mse_host, tq_encode,
                      tq_outlier_channels, tq_prepare_queries, tq_qjl_matrix, tq_rerank, tq_score,
                      tq_score_prepare, tq_score_prepared, tq_selftest_timeout, tq_set_qjl_onthefly,
                      tq_sync_check, tq_topk)
