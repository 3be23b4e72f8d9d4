"""B200-native (sm_100a) QSA hot path: indexer scores -> exact Top-K -> expand -> sparse attention."""
