"""B200-native exact attention forward (sm_100a, tcgen05/TMEM/TMA)."""
