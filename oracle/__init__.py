"""fp64 CPU oracle (test infrastructure only; see rtp_oracle's header)."""

from .rtp_oracle import (IDX_DIM, INDEXER_SCALE, OracleCache, attend, decode, decode_recall, indexer_project,
                         indexer_scores, prefill, recall_of_rows, rope, rope_inv_freq, round_bf16,
                         round_storage,
                         sink_window_set, top_k_set, top_p_set)

__all__ = ["IDX_DIM", "INDEXER_SCALE", "OracleCache", "attend", "decode", "decode_recall", "indexer_project",
           "indexer_scores", "prefill", "recall_of_rows", "rope", "rope_inv_freq", "round_bf16", "round_storage",
           "sink_window_set", "top_k_set", "top_p_set"]
