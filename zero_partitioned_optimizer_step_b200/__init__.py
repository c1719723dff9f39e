"""B200-native ZeRO partitioned optimizer step (package placeholder)."""
