"""Spark FFN with statistical top-k on B200 (sm_100a)."""
