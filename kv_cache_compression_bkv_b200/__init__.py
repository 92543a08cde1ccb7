"""B200-native BeaconKV KV-cache compression step."""
