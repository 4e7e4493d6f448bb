"""Low-rank compressed-KV decode attention on B200 (placeholder; binding follows)."""
